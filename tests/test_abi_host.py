"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/w4a16.h declares, and rejects bad arguments
before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a16_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from conftest import build_library
    build_library()
    import weight_only_int4_a16w4_b200 as w4
    return w4


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("w4a16_repack", "w4a16_msd_matmul", "w4a16_dequant_matmul", "w4a16_grouped_matmul",
              "w4a16_msd_debug_yint", "w4a16_workspace_size", "w4a16_packed_bytes",
              "w4a16_dequant_matmul_bf16", "w4a16_moe_combine_bf16"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(so, name), name
        # the binding exposes the same names
        assert hasattr(lib, name), name


def test_packed_bytes(lib):
    assert lib.w4a16_packed_bytes(4096, 4096) == 4096 * 4096 // 2
    assert lib.w4a16_packed_bytes(4096, 14336) == 4096 * 14336 // 2
    assert lib.w4a16_packed_bytes(192, 136) == 2 * 2 * 8192       # padded to 128 x 128 tiles
    assert lib.w4a16_packed_bytes(0, 8) == 0


def test_workspace_sizes(lib):
    msd = lib.w4a16_workspace_size(lib.OP_MSD, 16, 4096, 14336, 128)
    deq = lib.w4a16_workspace_size(lib.OP_DEQUANT, 16, 4096, 14336, 128)
    # MSD holds A_int (3*M*K bytes) and A_max (K/g*M floats) on top of what DEQUANT needs
    assert msd - deq >= 3 * 16 * 4096 + 32 * 16 * 4
    assert lib.w4a16_workspace_size(lib.OP_DEQUANT, 0, 256, 256, 64) >= 256
    assert lib.w4a16_workspace_size(lib.OP_MSD, 4096, 4096, 14336, 128, E=8) >= 3 * 4096 * 4096
    # MSD with S unfold steps holds S digit planes (S * M * K bytes)
    m2, m3, m4 = (lib.w4a16_workspace_size(op, 4096, 4096, 4096, 128)
                  for op in (lib.OP_MSD_2STEP, lib.OP_MSD, lib.OP_MSD_4STEP))
    assert m3 - m2 == 4096 * 4096 and m4 - m3 == 4096 * 4096
    # the bf16 dequant variant needs what the fp16 one needs
    for M in (1, 8, 16, 4096):
        assert lib.w4a16_workspace_size(lib.OP_DEQUANT_BF16, M, 4096, 14336, 128) == \
            lib.w4a16_workspace_size(lib.OP_DEQUANT, M, 4096, 14336, 128)


@pytest.mark.parametrize("args,code", [
    ((0, 16, 4096, 4100, 128), 1),      # N % 8 != 0
    ((0, 16, 4000, 4096, 128), 1),      # K % g != 0
    ((0, 16, 3840, 4096, 96), 2),       # g = 96 unsupported
    ((0, -1, 4096, 4096, 128), 1),      # negative M
    ((0, 16, 4096, 4096, 1024), 2),     # MSD group larger than 512
    ((7, 16, 4096, 4096, 128), 1),      # bad op
    ((5, 16, 4096, 4096, 128), 1),      # first code past the MSD step variants
    ((4, 16, 4096, 4096, 1024), 2),     # four-step MSD, group larger than 512
])
def test_workspace_size_rejects(lib, args, code):
    with pytest.raises(lib.W4A16Error) as e:
        lib.w4a16_workspace_size(*args)
    assert e.value.code == code


def test_matmul_rejects_before_launch(lib):
    fake = 1 << 40                       # 16-byte aligned, never dereferenced
    for fn in (lib.w4a16_msd_matmul, lib.w4a16_dequant_matmul, lib.w4a16_dequant_matmul_bf16):
        with pytest.raises(lib.W4A16Error) as e:     # null x
            fn(None, fake, fake, 16, 256, 256, 64, fake, fake, 1 << 20, stream=0)
        assert e.value.code == 1
        with pytest.raises(lib.W4A16Error) as e:     # misaligned y
            fn(fake, fake, fake, 16, 256, 256, 64, fake + 2, fake, 1 << 20, stream=0)
        assert e.value.code == 1
        with pytest.raises(lib.W4A16Error) as e:     # workspace too small
            fn(fake, fake, fake, 16, 256, 256, 64, fake, fake, 16, stream=0)
        assert e.value.code == 3
        with pytest.raises(lib.W4A16Error) as e:     # unsupported group
            fn(fake, fake, fake, 16, 288, 256, 96, fake, fake, 1 << 20, stream=0)
        assert e.value.code == 2
    # M == 0 is a no-op that touches nothing
    lib.w4a16_dequant_matmul(None, None, None, 0, 256, 256, 64, None, None, 0, stream=0)
    # MSD unfold steps other than 2, 3, 4 are rejected
    for steps in (0, 1, 5):
        with pytest.raises(lib.W4A16Error) as e:
            lib.w4a16_msd_matmul_steps(steps, fake, fake, fake, 16, 256, 256, 64, fake, fake, 1 << 20, stream=0)
        assert e.value.code == 1
    with pytest.raises(lib.W4A16Error) as e:     # workspace sized for 3 steps is too small for 4
        need = lib.w4a16_workspace_size(lib.OP_MSD, 64, 256, 256, 64)
        lib.w4a16_msd_matmul_steps(4, fake, fake, fake, 64, 256, 256, 64, fake, fake, need, stream=0)
    assert e.value.code == 3


def test_grouped_and_debug_reject(lib):
    fake = 1 << 40
    with pytest.raises(lib.W4A16Error) as e:         # too many experts
        lib.w4a16_grouped_matmul(0, fake, [fake] * 65, [fake] * 65, fake, 65, 64, 256, 256, 64, fake, fake,
                                 1 << 30, stream=0)
    assert e.value.code == 1
    with pytest.raises(lib.W4A16Error) as e:         # null expert weight
        lib.w4a16_grouped_matmul(1, fake, [fake, None], [fake, fake], fake, 2, 64, 256, 256, 64, fake, fake,
                                 1 << 30, stream=0)
    assert e.value.code == 1
    with pytest.raises(lib.W4A16Error) as e:         # empty debug window
        lib.w4a16_msd_debug_yint(fake, fake, 16, 256, 256, 64, 3, 3, 0, 8, fake, fake, fake, 1 << 20,
                                 stream=0)
    assert e.value.code == 1


def test_repack_rejects(lib):
    fake = 1 << 40
    with pytest.raises(lib.W4A16Error):
        lib.w4a16_repack(fake, 255, 256, fake, stream=0)     # odd K
    with pytest.raises(lib.W4A16Error):
        lib.w4a16_repack(fake, 256, 250, fake, stream=0)     # N % 8
    with pytest.raises(lib.W4A16Error):
        lib.w4a16_repack(fake, 256, 256, fake + 8, stream=0)  # misaligned output


def test_moe_entry_points_reject_before_launch(lib):
    fake = 1 << 40
    cases = [
        (lambda: lib.w4a16_moe_align(fake, 4, 2, 0, fake, fake, fake, fake, 1 << 20, stream=0), 1),    # E = 0
        (lambda: lib.w4a16_moe_align(fake, 4, 2, 65, fake, fake, fake, fake, 1 << 20, stream=0), 1),   # E > 64
        (lambda: lib.w4a16_moe_align(fake, 4, 0, 8, fake, fake, fake, fake, 1 << 20, stream=0), 1),    # topk = 0
        (lambda: lib.w4a16_moe_align(fake, 4, 2, 8, fake, fake, fake, fake, 16, stream=0), 3),         # workspace
        (lambda: lib.w4a16_moe_gather(fake, fake, 4, 12, fake, stream=0), 1),                          # K % 8
        (lambda: lib.w4a16_moe_gather(fake + 8, fake, 4, 16, fake, stream=0), 1),                      # misaligned x
        (lambda: lib.w4a16_moe_combine(fake, fake, fake, 4, 2, 20, fake, stream=0), 1),                # N % 8
        (lambda: lib.w4a16_moe_combine(fake, None, fake, 4, 2, 16, fake, stream=0), 1),                # null inv_pos
        (lambda: lib.w4a16_moe_combine_bf16(fake + 4, fake, fake, 4, 2, 16, fake, stream=0), 1),       # misaligned rows
        (lambda: lib.w4a16_moe_workspace_size(0, 4, 2, 576, 256, 96, 8), 2),                           # g = 96
    ]
    for fn, code in cases:
        with pytest.raises(lib.W4A16Error) as e:
            fn()
        assert e.value.code == code
    # empty inputs are no-ops that touch nothing
    lib.w4a16_moe_gather(None, None, 0, 16, None, stream=0)
    lib.w4a16_moe_combine(None, None, None, 0, 2, 16, None, stream=0)


def test_moe_workspace_holds_every_intermediate(lib):
    T, topk, K, N, g, E = 100, 2, 512, 264, 64, 8
    total = lib.w4a16_moe_workspace_size(1, T, topk, K, N, g, E)
    grouped = lib.w4a16_workspace_size(1, T * topk, K, N, g, E)
    assert total >= grouped + (E + 1) * 4 + 2 * T * topk * 4 + T * topk * (K + N) * 2


def test_binding_constants_match_the_header(lib):
    """The op codes, device status bits and status codes the binding exposes
    are the header's values."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    consts = {k: int(v.rstrip("u")) for k, v in re.findall(r"\b(W4A16_[A-Z0-9_]+)\s*=\s*([0-9]+u?)", text)}
    for name in ("OP_MSD", "OP_DEQUANT", "OP_DEQUANT_BF16", "OP_MSD_2STEP", "OP_MSD_4STEP",
                 "DEVICE_TIMEOUT", "DEVICE_BAD_EXPERT"):
        assert getattr(lib, name) == consts["W4A16_" + name], name
    for code, name in lib._STATUS_NAMES.items():
        assert consts[name] == code, name
    # the allocation-free entry point's array size, a macro of the form (a << b)
    m = re.search(r"#define\s+W4A16_NOALLOC_SCRATCH_BYTES\s+\((\d+)u?\s*<<\s*(\d+)\)", text)
    assert m, "W4A16_NOALLOC_SCRATCH_BYTES not found in the header"
    assert lib.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_is_plain_c_and_cxx(lang, std, tmp_path):
    """The ABI header compiles on its own as C99 (no C++ or CUDA types leak
    into it) and as C++11, warning-free; a C translation unit can call every
    entry point with plain pointers."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / ("use." + ("c" if lang == "c" else "cpp"))
    src.write_text('#include "w4a16.h"\n'
                   "int main(void) {\n"
                   "    size_t ws = 0;\n"
                   "    w4a16_status s = w4a16_workspace_size(W4A16_OP_MSD, 1, 256, 256, 128, 1, &ws);\n"
                   "    return (int)s + (int)w4a16_packed_bytes(256, 256) * 0;\n"
                   "}\n")
    r = subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
