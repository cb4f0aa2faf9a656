"""Python binding of libw4a16.so, the B200 (sm_100a) A16W4 per-group matmul.

The functions below carry the names of the C ABI in ``include/w4a16.h`` and
only marshal arguments (torch CUDA tensors -> device pointers, the current
torch stream -> cudaStream_t); every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback: importing this package
fails loudly when the library has not been built.

Operator: y = x . (antiquant_scale (.) W) -- "WeightQuantBatchMatmulExperiment
算子深度解析" (bjdmk.com.cn/news/4847346), sections 4.1-4.3.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("W4A16_LIBRARY") or os.path.join(_PKG, "libw4a16.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python weight_only_int4_a16w4_b200/build.py` "
        "(nvcc, sm_100a); this package has no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

OP_MSD = 0
OP_DEQUANT = 1
OP_DEQUANT_BF16 = 2
OP_MSD_2STEP = 3
OP_MSD_4STEP = 4
DEVICE_TIMEOUT = 1
DEVICE_BAD_EXPERT = 2

_STATUS_NAMES = {0: "W4A16_OK", 1: "W4A16_ERR_INVALID_ARG", 2: "W4A16_ERR_UNSUPPORTED",
                 3: "W4A16_ERR_WORKSPACE", 4: "W4A16_ERR_CUDA", 5: "W4A16_ERR_TIMEOUT",
                 6: "W4A16_ERR_BAD_INDEX"}


class W4A16Error(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        msg = _lib.w4a16_status_string(code).decode()
        super().__init__(f"{where}: {_STATUS_NAMES.get(code, code)} ({msg})")


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_lib.w4a16_status_string.restype = ctypes.c_char_p
_lib.w4a16_status_string.argtypes = [_I]
_lib.w4a16_packed_bytes.restype = _SZ
_lib.w4a16_packed_bytes.argtypes = [_I, _I]
_lib.w4a16_workspace_size.restype = _I
_lib.w4a16_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]
_lib.w4a16_repack.restype = _I
_lib.w4a16_repack.argtypes = [_P, _I, _I, _P, _P]
for _name in ("w4a16_msd_matmul", "w4a16_dequant_matmul", "w4a16_dequant_matmul_bf16"):
    getattr(_lib, _name).restype = _I
    getattr(_lib, _name).argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.w4a16_grouped_matmul.restype = _I
_lib.w4a16_grouped_matmul.argtypes = [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.w4a16_msd_matmul_steps.restype = _I
_lib.w4a16_msd_matmul_steps.argtypes = [_I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.w4a16_msd_debug_yint_steps.restype = _I
_lib.w4a16_msd_debug_yint_steps.argtypes = [_I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]
_lib.w4a16_msd_debug_yint.restype = _I
_lib.w4a16_msd_debug_yint.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]
_lib.w4a16_msd_matmul_noalloc.restype = _I
_lib.w4a16_msd_matmul_noalloc.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.w4a16_moe_align.restype = _I
_lib.w4a16_moe_align.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]
_lib.w4a16_moe_gather.restype = _I
_lib.w4a16_moe_gather.argtypes = [_P, _P, _I, _I, _P, _P]
for _name in ("w4a16_moe_combine", "w4a16_moe_combine_bf16"):
    getattr(_lib, _name).restype = _I
    getattr(_lib, _name).argtypes = [_P, _P, _P, _I, _I, _I, _P, _P]
_lib.w4a16_moe_workspace_size.restype = _I
_lib.w4a16_moe_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]
_lib.w4a16_moe_matmul.restype = _I
_lib.w4a16_moe_matmul.argtypes = [_I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.w4a16_read_status.restype = _I
_lib.w4a16_read_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]
_lib.w4a16_set_wait_timeout_ns.restype = None
_lib.w4a16_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
_lib.w4a16_selftest_wait_timeout.restype = _I
_lib.w4a16_selftest_wait_timeout.argtypes = [_P, ctypes.c_uint64, _P]


def library():
    """The loaded ctypes library (for tests that check its exports)."""
    return _lib


def _ptr(t):
    """Device (or host) address of a tensor, an int address, or None -> NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code, where):
    if code != 0:
        raise W4A16Error(code, where)


def w4a16_packed_bytes(K: int, N: int) -> int:
    return int(_lib.w4a16_packed_bytes(K, N))


def w4a16_workspace_size(op: int, M: int, K: int, N: int, group_size: int, E: int = 1) -> int:
    out = _SZ(0)
    _check(_lib.w4a16_workspace_size(op, M, K, N, group_size, E, ctypes.byref(out)),
           "w4a16_workspace_size")
    return int(out.value)


def w4a16_repack(w_logical, K: int, N: int, w_packed, stream=None):
    _check(_lib.w4a16_repack(_ptr(w_logical), K, N, _ptr(w_packed), _stream(stream)), "w4a16_repack")


def w4a16_msd_matmul(x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes=None,
                     stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_msd_matmul(_ptr(x), _ptr(w_packed), _ptr(scale), M, K, N, group_size, _ptr(y),
                                 _ptr(workspace), wb, _stream(stream)), "w4a16_msd_matmul")


def w4a16_dequant_matmul(x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes=None,
                         stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_dequant_matmul(_ptr(x), _ptr(w_packed), _ptr(scale), M, K, N, group_size, _ptr(y),
                                     _ptr(workspace), wb, _stream(stream)), "w4a16_dequant_matmul")


def w4a16_dequant_matmul_bf16(x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes=None,
                              stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_dequant_matmul_bf16(_ptr(x), _ptr(w_packed), _ptr(scale), M, K, N, group_size, _ptr(y),
                                          _ptr(workspace), wb, _stream(stream)), "w4a16_dequant_matmul_bf16")


def w4a16_grouped_matmul(op, x, w_packed_list, scale_list, offsets, E, T, K, N, group_size, y, workspace,
                         workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    wp = (ctypes.c_void_p * E)(*[_ptr(t) for t in w_packed_list])
    sp = (ctypes.c_void_p * E)(*[_ptr(t) for t in scale_list])
    _check(_lib.w4a16_grouped_matmul(op, _ptr(x), ctypes.cast(wp, _P), ctypes.cast(sp, _P), _ptr(offsets), E,
                                     T, K, N, group_size, _ptr(y), _ptr(workspace), wb, _stream(stream)),
           "w4a16_grouped_matmul")


def w4a16_msd_debug_yint(x, w_packed, M, K, N, group_size, m0, m1, n0, n1, yint, amax, workspace,
                         workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_msd_debug_yint(_ptr(x), _ptr(w_packed), M, K, N, group_size, m0, m1, n0, n1, _ptr(yint),
                                     _ptr(amax), _ptr(workspace), wb, _stream(stream)),
           "w4a16_msd_debug_yint")


def w4a16_msd_matmul_steps(steps, x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes=None,
                           stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_msd_matmul_steps(steps, _ptr(x), _ptr(w_packed), _ptr(scale), M, K, N, group_size, _ptr(y),
                                       _ptr(workspace), wb, _stream(stream)), "w4a16_msd_matmul_steps")


def w4a16_msd_debug_yint_steps(steps, x, w_packed, M, K, N, group_size, m0, m1, n0, n1, yint, amax, workspace,
                               workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_msd_debug_yint_steps(steps, _ptr(x), _ptr(w_packed), M, K, N, group_size, m0, m1, n0, n1,
                                           _ptr(yint), _ptr(amax), _ptr(workspace), wb, _stream(stream)),
           "w4a16_msd_debug_yint_steps")


def w4a16_moe_align(topk_ids, T, topk, E, offsets, sorted_token, inv_pos, workspace, workspace_bytes=None,
                    stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(_lib.w4a16_moe_align(_ptr(topk_ids), T, topk, E, _ptr(offsets), _ptr(sorted_token), _ptr(inv_pos),
                                _ptr(workspace), wb, _stream(stream)), "w4a16_moe_align")


def w4a16_moe_gather(x, sorted_token, rows, K, x_sorted, stream=None):
    _check(_lib.w4a16_moe_gather(_ptr(x), _ptr(sorted_token), rows, K, _ptr(x_sorted), _stream(stream)),
           "w4a16_moe_gather")


def w4a16_moe_combine(y_sorted, inv_pos, topk_weights, T, topk, N, y, stream=None):
    _check(_lib.w4a16_moe_combine(_ptr(y_sorted), _ptr(inv_pos), _ptr(topk_weights), T, topk, N, _ptr(y),
                                  _stream(stream)), "w4a16_moe_combine")


def w4a16_moe_combine_bf16(y_sorted, inv_pos, topk_weights, T, topk, N, y, stream=None):
    _check(_lib.w4a16_moe_combine_bf16(_ptr(y_sorted), _ptr(inv_pos), _ptr(topk_weights), T, topk, N, _ptr(y),
                                       _stream(stream)), "w4a16_moe_combine_bf16")


def w4a16_moe_workspace_size(op, T, topk, K, N, group_size, E) -> int:
    out = _SZ(0)
    _check(_lib.w4a16_moe_workspace_size(op, T, topk, K, N, group_size, E, ctypes.byref(out)),
           "w4a16_moe_workspace_size")
    return int(out.value)


def w4a16_moe_matmul(op, x, topk_ids, topk_weights, w_packed_list, scale_list, E, T, topk, K, N, group_size, y,
                     workspace, workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    wp = (ctypes.c_void_p * E)(*[_ptr(t) for t in w_packed_list])
    sp = (ctypes.c_void_p * E)(*[_ptr(t) for t in scale_list])
    _check(_lib.w4a16_moe_matmul(op, _ptr(x), _ptr(topk_ids), _ptr(topk_weights), ctypes.cast(wp, _P),
                                 ctypes.cast(sp, _P), E, T, topk, K, N, group_size, _ptr(y), _ptr(workspace), wb,
                                 _stream(stream)), "w4a16_moe_matmul")


NOALLOC_SCRATCH_BYTES = 8 << 20


def w4a16_msd_matmul_noalloc(x, w_packed, scale, M, K, N, group_size, y, stream=None):
    """MSD matmul whose scratch lives in the library's own device array (no
    workspace argument; for callers that cannot allocate device memory)."""
    _check(_lib.w4a16_msd_matmul_noalloc(_ptr(x), _ptr(w_packed), _ptr(scale), M, K, N, group_size, _ptr(y),
                                         _stream(stream)), "w4a16_msd_matmul_noalloc")


def w4a16_read_status(workspace, stream=None) -> int:
    """Device status word of a workspace (synchronises the stream)."""
    out = ctypes.c_uint32(0)
    code = _lib.w4a16_read_status(_ptr(workspace), _stream(stream), ctypes.byref(out))
    if code not in (0, 5, 6):
        _check(code, "w4a16_read_status")
    return int(out.value)


def w4a16_set_wait_timeout_ns(ns: int):
    _lib.w4a16_set_wait_timeout_ns(int(ns))


def w4a16_selftest_wait_timeout(workspace, timeout_ns: int, stream=None):
    _check(_lib.w4a16_selftest_wait_timeout(_ptr(workspace), int(timeout_ns), _stream(stream)),
           "w4a16_selftest_wait_timeout")


# ---------------------------------------------------------------- conveniences

def alloc_workspace(op, M, K, N, group_size, E=1, device="cuda"):
    """Zero-filled workspace of the size the call needs (the library itself never allocates)."""
    import torch
    nbytes = w4a16_workspace_size(op, M, K, N, group_size, E)
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def repack(w_logical, K, N, stream=None):
    """Packed kernel-layout copy of logical int4 bytes [K/2, N] (a new device tensor)."""
    import torch
    out = torch.empty(w4a16_packed_bytes(K, N), dtype=torch.uint8, device=w_logical.device)
    w4a16_repack(w_logical, K, N, out, stream)
    return out


def w4a16_status_string(code: int) -> str:
    return _lib.w4a16_status_string(int(code)).decode()
