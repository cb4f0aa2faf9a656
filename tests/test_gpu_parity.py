"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs.

Bars (from the method's acceptance rules):
  * MSD equation 9: the per-group int32 Y1, Y2, Y3 (debug window) and A_max
    are bit-exact against the oracle's.
  * MSD y: |y - y_oracle| <= 2e-3 * max|y_oracle| + 1e-3, y_oracle the
    binary64 result of equations 1-11.
  * DEQUANT y: ||y - y_exact||_F / ||y_exact||_F <= 1e-3 against the exact
    binary64 GEMM.
Full-size workloads are checked on sampled outputs the oracle computes one
by one, in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest

import oracle
from inputs import make_case, make_workload, pack_int4

pytestmark = pytest.mark.gpu

MSD_REL, MSD_ABS = 2e-3, 1e-3
DEQ_REL_F = 1e-3


def _t():
    import torch
    return torch


def upload(w4, c):
    torch = _t()
    dev = {"x": torch.from_numpy(c.x).cuda()}
    dev["wp"] = [w4.repack(torch.from_numpy(wp).cuda(), c.K, c.N) for wp in c.wp]
    dev["scale"] = [torch.from_numpy(s).cuda() for s in c.scale]
    if c.offsets is not None:
        dev["offsets"] = torch.from_numpy(c.offsets).cuda()
    return dev


def run_dense(w4, op, c, dev, ws=None):
    torch = _t()
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.float16, device="cuda")
    if ws is None:
        ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g)
    fn = w4.w4a16_msd_matmul if op == w4.OP_MSD else w4.w4a16_dequant_matmul
    fn(dev["x"], dev["wp"][0], dev["scale"][0], c.M, c.K, c.N, c.g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.cpu().numpy().astype(np.float64)


def run_grouped(w4, op, c, dev):
    torch = _t()
    T = c.M
    y = torch.full((T, c.N), float("nan"), dtype=torch.float16, device="cuda")
    ws = w4.alloc_workspace(op, T, c.K, c.N, c.g, E=c.E)
    w4.w4a16_grouped_matmul(op, dev["x"], dev["wp"], dev["scale"], dev["offsets"], c.E, T, c.K, c.N, c.g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.cpu().numpy().astype(np.float64)


def assert_msd_close(y, ref, what=""):
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    tol = MSD_REL * np.abs(ref).max() + MSD_ABS
    err = np.abs(y - ref)
    i = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= tol, f"{what}: max err {err.max():.3e} at {i} (gpu {y[i]}, oracle {ref[i]}), tol {tol:.3e}"


def assert_deq_close(y, ref, what=""):
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    rel = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= DEQ_REL_F, f"{what}: relative Frobenius error {rel:.3e}"


def debug_yint(w4, c, dev, m0, m1, n0, n1):
    torch = _t()
    G = c.K // c.g
    yint = torch.full((3, m1 - m0, G, n1 - n0), -12345, dtype=torch.int32, device="cuda")
    amax = torch.full((m1 - m0, G), -1.0, dtype=torch.float32, device="cuda")
    ws = w4.alloc_workspace(w4.OP_MSD, c.M, c.K, c.N, c.g)
    w4.w4a16_msd_debug_yint(dev["x"], dev["wp"][0], c.M, c.K, c.N, c.g, m0, m1, n0, n1, yint, amax, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return yint.cpu().numpy(), amax.cpu().numpy()


def check_yint(w4, c, dev, m0, m1, n0, n1):
    yint, amax = debug_yint(w4, c, dev, m0, m1, n0, n1)
    ref_amax, a = oracle.msd_expand(c.x[m0:m1], c.g)
    ref = oracle.msd_yint(a, np.ascontiguousarray(c.wp[0][:, n0:n1]), n1 - n0, c.g)
    assert np.array_equal(amax.astype(np.float64), ref_amax), "A_max differs"
    bad = np.argwhere(yint.astype(np.int64) != ref)
    assert bad.size == 0, f"{len(bad)} Y_int mismatches, first at {bad[0]}: gpu {yint[tuple(bad[0])]} " \
                          f"oracle {ref[tuple(bad[0])]}"


# ---------------------------------------------------------------- failure path

def test_bounded_wait_reports_timeout(cuda_lib):
    torch = _t()
    w4 = cuda_lib
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    w4.w4a16_selftest_wait_timeout(ws, 2_000_000)       # 2 ms on a barrier nothing completes
    assert w4.w4a16_read_status(ws) == w4.DEVICE_TIMEOUT
    # the context is still usable
    c = make_case(16, 256, 256, 64, seed=3)
    dev = upload(w4, c)
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], 64))


# ---------------------------------------------------------------- small shapes, full comparison

SMALL = [
    # (M, K, N, g)                       what it covers
    (16, 256, 256, 64),                  # the 16x256x256 workload shape
    (1, 256, 128, 128),                  # one row, one tile
    (5, 384, 136, 64),                   # ragged N (136 = 128 + 8), 3 K chunks
    (16, 192, 256, 64),                  # K not a multiple of 128
    (3, 512, 256, 256),                  # group spanning two K chunks
    (9, 512, 384, 32),                   # four groups per K chunk
    (17, 256, 264, 128),                 # first M above the decode tile
    (70, 512, 256, 64),                  # several token tiles, ragged tail
    (130, 384, 520, 128),                # ragged in every dimension
]


@pytest.mark.parametrize("M,K,N,g", SMALL)
def test_msd_small(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 7919 + K * 31 + N + g)
    if M > 3:
        c.x[3, :g] = 0                   # an all-zero group
    dev = upload(w4, c)
    y = run_dense(w4, w4.OP_MSD, c, dev)
    assert_msd_close(y, oracle.msd(c.x, c.wp[0], c.scale[0], g), f"msd {M}x{K}x{N} g{g}")


@pytest.mark.parametrize("M,K,N,g", SMALL)
def test_dequant_small(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 7919 + K * 31 + N + g + 1)
    dev = upload(w4, c)
    y = run_dense(w4, w4.OP_DEQUANT, c, dev)
    assert_deq_close(y, oracle.dequant(c.x, c.wp[0], c.scale[0], g), f"dequant {M}x{K}x{N} g{g}")


@pytest.mark.parametrize("M,K,N,g", [(16, 256, 256, 64), (5, 384, 136, 64), (3, 512, 256, 256),
                                     (9, 512, 384, 32), (70, 512, 256, 64), (6, 768, 264, 384)])
def test_msd_yint_bit_exact(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=99 + M + g)
    c.x[0, :g] = np.float16(-2.5)        # every entry equals -A_max
    if M > 2:
        c.x[2] *= np.float16(1e-4)       # tiny values
    dev = upload(w4, c)
    check_yint(w4, c, dev, 0, M, 0, N)


def test_page_example_distributions(cuda_lib):
    """The page's own example distributions (x, scale ~ U[-3,3], w in [-7,7]),
    at a reduced K so the full oracle is quick; negative scales included."""
    from inputs import page_example
    w4 = cuda_lib
    c = page_example(M=4, K=1024, N=1536)
    dev = upload(w4, c)
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], c.g), "msd")
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], c.g),
                     "dequant")


def test_zero_rows_is_noop(cuda_lib):
    torch = _t()
    w4 = cuda_lib
    y = torch.zeros(4, dtype=torch.float16, device="cuda")
    w4.w4a16_msd_matmul(None, None, None, 0, 256, 256, 64, y, None, 0)
    w4.w4a16_dequant_matmul(None, None, None, 0, 256, 256, 64, y, None, 0)
    torch.cuda.synchronize()
    assert not y.any()


def test_repeat_calls_are_deterministic(cuda_lib):
    """The split-K partials meet in a fixed (rank) order on chip: the
    same bits on every call."""
    torch = _t()
    w4 = cuda_lib
    c = make_case(16, 2048, 1024, 128, seed=1234)
    dev = upload(w4, c)
    for op in (w4.OP_MSD, w4.OP_DEQUANT):
        ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g)
        ys = [run_dense(w4, op, c, dev, ws) for _ in range(3)]
        assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[1], ys[2])
    torch.cuda.synchronize()


# ---------------------------------------------------------------- decode GEMVs

# Small-M shapes (the CUDA-core GEMV, the warp-MMA GEMV or the decode tile,
# whichever the dispatch picks): every group size, ragged N and K, and work
# splits where many CTAs share one column tile (N small, K long) or one CTA
# spans two tiles (N large, K short).
GEMV = [
    # (M, K, N, g)                       what it covers
    (1, 4096, 136, 128),                 # 2 tiles x 32 chunks: ~32 CTAs add into each tile
    (2, 256, 14336, 64),                 # 224 blocks over the SMs: CTAs straddle tile edges
    (3, 1280, 520, 32),                  # four groups per chunk, ragged N, M below the row template
    (4, 768, 1032, 256),                 # group spanning two chunks, ragged N
    (1, 2560, 392, 512),                 # group of 512 (four chunks), K = 5 groups
    (4, 8192, 264, 128),                 # the largest M * K the kernel takes
    (2, 96, 128, 32),                    # K shorter than one chunk
]


@pytest.mark.parametrize("M,K,N,g", GEMV)
def test_gemv_msd(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 131 + K * 7 + N * 3 + g)
    c.x[M - 1, :g] = 0                   # an all-zero group
    dev = upload(w4, c)
    y = run_dense(w4, w4.OP_MSD, c, dev)
    assert_msd_close(y, oracle.msd(c.x, c.wp[0], c.scale[0], g), f"gemv msd {M}x{K}x{N} g{g}")


@pytest.mark.parametrize("M,K,N,g", GEMV)
def test_gemv_dequant(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 137 + K * 5 + N * 11 + g)
    dev = upload(w4, c)
    y = run_dense(w4, w4.OP_DEQUANT, c, dev)
    assert_deq_close(y, oracle.dequant(c.x, c.wp[0], c.scale[0], g), f"gemv dequant {M}x{K}x{N} g{g}")


# Decode-sized shapes for both variants (the CUDA-core GEMV at M <= 4, the
# tensor-core decode tile above): every group size including 384 (groups
# that cut 128-deep chunks), ragged N, K not a multiple of 1024 or of 128,
# one and several column blocks per CTA.
DECODE = [
    # (M, K, N, g)                       what it covers
    (7, 1536, 264, 64),                  # odd M, partial stage, ragged N
    (12, 3072, 520, 384),                # group of 384 (stages cut groups), 3 stages
    (4, 1152, 776, 384),                 # MSD with 3 sub-chunks per span, partial last stage
    (3, 8192, 96, 512),                  # 8 stages, one tile, N = 3 blocks
    (1, 640, 4104, 32),                  # 129 column blocks over the SMs, ragged last block
    (2, 160, 520, 32),                   # K of 5 pieces (not a multiple of 128)
    (16, 1024, 2048, 128),               # the full 16 MMA rows, exactly one stage
    (5, 2048, 18432, 64),                # several column blocks per CTA
]


@pytest.mark.parametrize("M,K,N,g", DECODE)
def test_decode_shapes_both_variants(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 1009 + K * 13 + N * 7 + g)
    c.x[M - 1, g:2 * g] = 0              # an all-zero group
    dev = upload(w4, c)
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], g),
                     f"decode msd {M}x{K}x{N} g{g}")
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], g),
                     f"decode dequant {M}x{K}x{N} g{g}")


# Shapes that take the warp-MMA GEMV (dequant: g % 128 == 0, M <= 8; MSD:
# M <= 2 and K >= 2N): rows up to the full lower half of the m16 tile,
# quads fewer than warps (idle warps), groups of 2-4 quads cut by the
# warps' K split, one column block per CTA, a CTA with several 4-block
# rounds and a ragged last one, a single 8-column block.
MMA_DEQ = [
    # (M, K, N, g)
    (5, 4096, 520, 128),
    (8, 1536, 264, 256),
    (3, 1152, 776, 384),
    (6, 2560, 14344, 512),
    (2, 128, 64, 128),
    (7, 8192, 8, 128),
    (1, 1024, 8200, 128),                # 32-warp instance (M <= 2, N >= 8192), ragged last block
    (2, 2048, 16384, 256),               # 32-warp instance, groups over two quads
]
MMA_MSD = [
    (1, 8192, 1024, 128),
    (2, 4096, 264, 256),
    (2, 3072, 136, 384),
    (1, 4096, 2048, 512),
    (2, 1152, 8, 128),
]


@pytest.mark.parametrize("M,K,N,g", MMA_DEQ)
def test_mma_gemv_dequant(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 313 + K * 17 + N * 5 + g)
    dev = upload(w4, c)
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], g),
                     f"mma dequant {M}x{K}x{N} g{g}")


@pytest.mark.parametrize("M,K,N,g", MMA_MSD)
def test_mma_gemv_msd(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 317 + K * 19 + N * 3 + g)
    c.x[M - 1, g:2 * g] = 0              # an all-zero group
    dev = upload(w4, c)
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], g),
                     f"mma msd {M}x{K}x{N} g{g}")


# Decode shapes between the GEMVs' row limits and 16 rows, g % 128 == 0
# (the tensor-core decode tile): few column tiles, K of two chunks, groups of
# 2-4 chunks, ragged N, the full 16 rows at the decode_m16 shape (sampled).
SK = [
    # (M, K, N, g)
    (9, 4096, 264, 128),
    (16, 1024, 64, 256),
    (5, 2560, 1032, 512),
    (16, 512, 4104, 128),
    (13, 256, 2048, 128),
    (3, 3072, 776, 384),
    (16, 4096, 14336, 128),
]


@pytest.mark.parametrize("M,K,N,g", SK)
def test_decode_tile_rows_both_variants(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 419 + K * 23 + N + g)
    c.x[M - 1, g:2 * g] = 0              # an all-zero group
    dev = upload(w4, c)
    if M * N > 20000:                    # the full oracle is slow here: sample
        rng = np.random.default_rng(M + N)
        rows = rng.integers(0, M, 3000)
        cols = rng.integers(0, N, 3000)
        ym = run_dense(w4, w4.OP_MSD, c, dev)[rows, cols]
        yd = run_dense(w4, w4.OP_DEQUANT, c, dev)[rows, cols]
        assert_msd_close(ym, oracle.msd_at(c.x, c.wp[0], c.scale[0], g, rows, cols), "decode msd sampled")
        ref_d = oracle.dequant_at(c.x, c.wp[0], c.scale[0], g, rows, cols)
        assert_deq_close(yd, ref_d, "decode dequant sampled")
        return
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], g),
                     f"decode msd {M}x{K}x{N} g{g}")
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], g),
                     f"decode dequant {M}x{K}x{N} g{g}")


def test_gemv_repeat_calls_are_deterministic(cuda_lib):
    """The warps' partial sums are added in warp order, so repeated calls on
    one workspace give the same bits."""
    w4 = cuda_lib
    c = make_case(1, 4096, 1032, 128, seed=77)
    dev = upload(w4, c)
    for op in (w4.OP_MSD, w4.OP_DEQUANT):
        ws = w4.alloc_workspace(op, c.M, c.K, c.N, c.g)
        ys = [run_dense(w4, op, c, dev, ws) for _ in range(4)]
        assert all(np.array_equal(ys[0], v) for v in ys[1:])


def test_gemv_page_example_distributions(cuda_lib):
    """The page's own value ranges (x, scale ~ U[-3, 3], w in [-7, 7]) at M = 1."""
    w4 = cuda_lib
    rng = np.random.default_rng(4847346)
    M, K, N, g = 1, 2048, 1536, 128
    x = rng.uniform(-3, 3, (M, K)).astype(np.float16)
    w = rng.integers(-7, 8, (K, N), dtype=np.int8)
    sc = rng.uniform(-3, 3, (K // g, N)).astype(np.float16)
    c = make_case(M, K, N, g, seed=1)
    c.x[:] = x
    c.wp[0] = pack_int4(w)
    c.scale[0] = sc
    dev = upload(w4, c)
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], sc, g), "gemv msd page")
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], sc, g), "gemv deq page")


# ---------------------------------------------------------------- grouped experts

def test_grouped_small_with_empty_experts(cuda_lib):
    w4 = cuda_lib
    c = make_case(150, 256, 264, 64, seed=4242, E=5)
    c.offsets[:] = [0, 40, 40, 41, 150, 150]         # empty, one-token and empty-last experts
    dev = upload(w4, c)
    ref_m = oracle.grouped("msd", c.x, c.wp, c.scale, c.offsets, c.g)
    ref_d = oracle.grouped("dequant", c.x, c.wp, c.scale, c.offsets, c.g)
    assert_msd_close(run_grouped(w4, w4.OP_MSD, c, dev), ref_m, "grouped msd")
    assert_deq_close(run_grouped(w4, w4.OP_DEQUANT, c, dev), ref_d, "grouped dequant")


# ---------------------------------------------------------------- full-size workloads

def _samples(rng, M, N, count):
    return rng.integers(0, M, count), rng.integers(0, N, count)


def _tile_samples(rng, M, N, tm, tn, extra=0):
    """One random (row, column) inside every tm x tn output tile (so a tile
    written to the wrong place, or not at all, is caught), plus `extra`
    uniform samples."""
    r0 = np.arange(0, M, tm)
    c0 = np.arange(0, N, tn)
    rr, cc = np.meshgrid(r0, c0, indexing="ij")
    rows = rr.ravel() + rng.integers(0, tm, rr.size)
    cols = cc.ravel() + rng.integers(0, tn, cc.size)
    rows, cols = np.minimum(rows, M - 1), np.minimum(cols, N - 1)
    if extra:
        er, ec = _samples(rng, M, N, extra)
        rows, cols = np.concatenate([rows, er]), np.concatenate([cols, ec])
    return rows, cols


def assert_all_finite(y, what):
    """The output starts as NaN: every element must have been written."""
    bad = np.argwhere(~np.isfinite(y))
    assert bad.size == 0, f"{what}: {len(bad)} outputs not written or not finite, first at {bad[0]}"


def test_workload_msd_small_full(cuda_lib):
    """16 x 256 x 256, g = 64, with the forced all-zero group."""
    w4 = cuda_lib
    c = make_workload(0)
    dev = upload(w4, c)
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], c.g), "msd")
    assert_deq_close(run_dense(w4, w4.OP_DEQUANT, c, dev), oracle.dequant(c.x, c.wp[0], c.scale[0], c.g),
                     "dequant")
    check_yint(w4, c, dev, 0, 16, 0, 256)


def test_workload_decode_m1_full(cuda_lib):
    """1 x 4096 x 4096, g = 128: every output checked, and Y1..Y3 and A_max
    bit-exact over every column and group -- through the kernels the
    benchmark times (the digit-record expansion and the warp-MMA GEMV)."""
    w4 = cuda_lib
    c = make_workload(1)
    dev = upload(w4, c)
    y = run_dense(w4, w4.OP_MSD, c, dev)
    assert_all_finite(y, "msd")
    assert_msd_close(y, oracle.msd(c.x, c.wp[0], c.scale[0], c.g), "msd")
    y = run_dense(w4, w4.OP_DEQUANT, c, dev)
    assert_all_finite(y, "dequant")
    assert_deq_close(y, oracle.dequant(c.x, c.wp[0], c.scale[0], c.g), "dequant")
    check_yint(w4, c, dev, 0, 1, 0, c.N)


def test_workload_decode_m16_sampled(cuda_lib):
    """16 x 4096 x 14336, g = 128: every output written, one sample in every
    16 x 128 tile plus 1024 more, and Y1..Y3 bit-exact on windows at both
    ends through the split-K decode tile the benchmark times (its cluster
    split and both epilogue groups)."""
    w4 = cuda_lib
    c = make_workload(2)
    dev = upload(w4, c)
    rng = np.random.default_rng(2)
    rows, cols = _tile_samples(rng, c.M, c.N, 16, 128, extra=1024)
    y = run_dense(w4, w4.OP_MSD, c, dev)
    assert_all_finite(y, "msd")
    assert_msd_close(y[rows, cols], oracle.msd_at(c.x, c.wp[0], c.scale[0], c.g, rows, cols), "msd")
    y = run_dense(w4, w4.OP_DEQUANT, c, dev)
    assert_all_finite(y, "dequant")
    assert_deq_close(y[rows, cols], oracle.dequant_at(c.x, c.wp[0], c.scale[0], c.g, rows, cols), "dequant")
    check_yint(w4, c, dev, 0, 16, 0, 264)
    check_yint(w4, c, dev, 0, 16, 14336 - 136, 14336)


def test_workload_prefill_sampled(cuda_lib):
    """4096 x 4096 x 4096, g = 128: every output written, one sample in every
    128 x 128 tile plus 1024 more, and a Y_int window."""
    w4 = cuda_lib
    c = make_workload(3)
    dev = upload(w4, c)
    rng = np.random.default_rng(3)
    rows, cols = _tile_samples(rng, c.M, c.N, 128, 128, extra=1024)
    y = run_dense(w4, w4.OP_MSD, c, dev)
    assert_all_finite(y, "msd")
    assert_msd_close(y[rows, cols], oracle.msd_at(c.x, c.wp[0], c.scale[0], c.g, rows, cols), "msd")
    y = run_dense(w4, w4.OP_DEQUANT, c, dev)
    assert_all_finite(y, "dequant")
    assert_deq_close(y[rows, cols], oracle.dequant_at(c.x, c.wp[0], c.scale[0], c.g, rows, cols), "dequant")
    check_yint(w4, c, dev, 4000, 4096, 4096 - 40, 4096)


def test_workload_moe_sampled(cuda_lib):
    """E = 8, T = 4096, K = 4096, N = 14336: every output written, one sample
    in every 64 x 128 tile plus 1024 more."""
    w4 = cuda_lib
    c = make_workload(4)
    dev = upload(w4, c)
    rng = np.random.default_rng(4)
    rows, cols = _tile_samples(rng, c.M, c.N, 64, 128, extra=1024)
    y = run_grouped(w4, w4.OP_MSD, c, dev)
    assert_all_finite(y, "moe msd")
    assert_msd_close(y[rows, cols], oracle.grouped_at("msd", c.x, c.wp, c.scale, c.offsets, c.g, rows, cols),
                     "moe msd")
    y = run_grouped(w4, w4.OP_DEQUANT, c, dev)
    assert_all_finite(y, "moe dequant")
    assert_deq_close(y[rows, cols],
                     oracle.grouped_at("dequant", c.x, c.wp, c.scale, c.offsets, c.g, rows, cols), "moe dequant")


# ---------------------------------------------------------------- Y_int through every decode branch

# (M, K, N, g, kernel the product call dispatches to for MSD)
YINT_BRANCHES = [
    (1, 4096, 4096, 128, "warp-MMA GEMV, one token"),
    (2, 2048, 1032, 256, "warp-MMA GEMV, two tokens, 256-deep groups cut between warps, ragged column blocks"),
    (1, 14336, 512, 128, "warp-MMA GEMV, several quads per warp"),
    (1, 1024, 4096, 64, "CUDA-core dp4a GEMV, g = 64"),
    (3, 2048, 520, 32, "CUDA-core dp4a GEMV, g = 32, three tokens"),
    (4, 4096, 4096, 128, "split-K decode tile (cluster of K ranges), four tokens"),
    (16, 4096, 2048, 128, "split-K decode tile, 16 tokens"),
    (9, 1024, 264, 64, "decode tile, g = 64, K split over a cluster of 8, ragged N"),
    (40, 512, 392, 128, "64-token tile, ragged tokens and columns"),
]


@pytest.mark.parametrize("M,K,N,g,branch", YINT_BRANCHES, ids=[b[4] for b in YINT_BRANCHES])
def test_yint_bit_exact_on_every_branch(cuda_lib, M, K, N, g, branch):
    """Equation 9's per-group int32 Y1..Y3 and A_max, bit-exact against the
    oracle, read back from the kernels the product MSD call runs for this
    shape (the debug window runs the same kernels and launch shapes), over
    every row, group and column."""
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=4100 + M + N)
    dev = upload(w4, c)
    check_yint(w4, c, dev, 0, M, 0, N)
    # and the product call on the same inputs is within the MSD bar
    assert_msd_close(run_dense(w4, w4.OP_MSD, c, dev), oracle.msd(c.x, c.wp[0], c.scale[0], g), branch)
