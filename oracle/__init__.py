"""CPU oracle for the A16W4 per-group matmul -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product.

The arithmetic lives in ``w4a16_oracle.c`` (plain C, binary64, with the MSD
expansion in IEEE binary32).  Each function follows the page
"WeightQuantBatchMatmulExperiment 算子深度解析" (bjdmk.com.cn/news/4847346),
section 4.1, equations 1-11; the dequant oracle is the plain definition
y = x . (antiquant_scale (.) W).  The readings taken where the page is silent
or garbled are listed at the top of the C file.

All arrays are numpy arrays: fp16 data is passed as ``np.float16`` (its bit
pattern is read by the C code), packed weights as ``uint8 [K/2, N]`` bytes
with the low nibble holding the even k (two's complement int4).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        lib.oracle_halves_to_double.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_doubles_to_half.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_unpack_w.argtypes = [P, I, I, P]
        lib.oracle_msd_expand.argtypes = [P, I, I, I, I, P, P]
        lib.oracle_msd_yint.argtypes = [P, P, I, I, I, I, P]
        lib.oracle_msd_combine.argtypes = [P, P, P, I, I, I, I, P]
        lib.oracle_msd.argtypes = [P, P, P, I, I, I, I, I, P]
        lib.oracle_msd_at.argtypes = [P, P, P, I, I, I, I, I, P, P, I, P]
        lib.oracle_msd_expand_steps.argtypes = [P, I, I, I, I, I, P, P]
        lib.oracle_msd_yint_planes.argtypes = [P, I, P, I, I, I, I, P]
        lib.oracle_msd_steps.argtypes = [P, P, P, I, I, I, I, I, I, P]
        lib.oracle_msd_at_steps.argtypes = [P, P, P, I, I, I, I, I, I, P, P, I, P]
        lib.oracle_dequant.argtypes = [P, P, P, I, I, I, I, P]
        lib.oracle_dequant_at.argtypes = [P, P, P, I, I, I, I, P, P, I, P]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16s_to_double.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_dequant_bf16.argtypes = [P, P, P, I, I, I, I, P]
        lib.oracle_moe_align.argtypes = [P, I, I, I, P, P, P]
        lib.oracle_moe_combine.argtypes = [P, P, P, I, I, I, P]
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


MODE_FP32 = 0   # binary32 expansion (the arithmetic the kernel constants fix)
MODE_FP64 = 1   # binary64 expansion (for the truncation-bound pin)


def num_threads() -> int:
    return _load().oracle_num_threads()


def half_to_double(h: np.ndarray) -> np.ndarray:
    h = _c(np.asarray(h, dtype=np.float16), np.float16)
    out = np.empty(h.shape, np.float64)
    _load().oracle_halves_to_double(_ptr(h), h.size, _ptr(out))
    return out


def double_to_half(v: np.ndarray) -> np.ndarray:
    v = _c(np.asarray(v, dtype=np.float64), np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_doubles_to_half(_ptr(v), v.size, _ptr(out))
    return out.view(np.float16)


def unpack_w(wp: np.ndarray, K: int, N: int) -> np.ndarray:
    """Logical packed bytes [K/2, N] -> int8 W [K, N]."""
    wp = _c(wp, np.uint8)
    assert wp.shape == (K // 2, N)
    w = np.empty((K, N), np.int8)
    _load().oracle_unpack_w(_ptr(wp), K, N, _ptr(w))
    return w


def msd_expand(x: np.ndarray, g: int, mode: int = MODE_FP32):
    """Equations 1-8: returns (amax [M, K/g] float64, a_int [3, M, K] int8)."""
    x = _c(x, np.float16)
    M, K = x.shape
    amax = np.empty((M, K // g), np.float64)
    a = np.empty((3, M, K), np.int8)
    _check(_load().oracle_msd_expand(_ptr(x), M, K, g, mode, _ptr(amax), _ptr(a)),
           "msd_expand")
    return amax, a


def msd_yint(a: np.ndarray, wp: np.ndarray, N: int, g: int) -> np.ndarray:
    """Equation 9 per group: Y_int [3, M, K/g, N] int64."""
    a = _c(a, np.int8)
    wp = _c(wp, np.uint8)
    _, M, K = a.shape
    y = np.empty((3, M, K // g, N), np.int64)
    _check(_load().oracle_msd_yint(_ptr(a), _ptr(wp), M, K, N, g, _ptr(y)), "msd_yint")
    return y


def msd_combine(yint: np.ndarray, amax: np.ndarray, scale: np.ndarray, K: int, g: int):
    """Equations 10-11 from stored Y_int: y [M, N] float64."""
    yint = _c(yint, np.int64)
    amax = _c(amax, np.float64)
    scale = _c(scale, np.float16)
    _, M, G, N = yint.shape
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_msd_combine(_ptr(yint), _ptr(amax), _ptr(scale), M, K, N, g,
                                      _ptr(y)), "msd_combine")
    return y


def msd(x: np.ndarray, wp: np.ndarray, scale: np.ndarray, g: int,
        mode: int = MODE_FP32) -> np.ndarray:
    """All eleven MSD steps: y [M, N] float64 (round with double_to_half)."""
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_msd(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g, mode, _ptr(y)),
           "msd")
    return y


def msd_expand_steps(x: np.ndarray, g: int, steps: int, mode: int = MODE_FP32):
    """Equations 1-8 with `steps` digits (reading R16 of the C file): returns
    (amax [M, K/g] float64, a_int [steps, M, K] int8)."""
    x = _c(x, np.float16)
    M, K = x.shape
    amax = np.empty((M, K // g), np.float64)
    a = np.empty((steps, M, K), np.int8)
    _check(_load().oracle_msd_expand_steps(_ptr(x), M, K, g, mode, steps, _ptr(amax), _ptr(a)),
           "msd_expand_steps")
    return amax, a


def msd_yint_planes(a: np.ndarray, wp: np.ndarray, N: int, g: int) -> np.ndarray:
    """Equation 9 per group for any number of digit planes: a [S, M, K] ->
    Y_int [S, M, K/g, N] int64."""
    a = _c(a, np.int8)
    wp = _c(wp, np.uint8)
    S, M, K = a.shape
    y = np.empty((S, M, K // g, N), np.int64)
    _check(_load().oracle_msd_yint_planes(_ptr(a), S, _ptr(wp), M, K, N, g, _ptr(y)), "msd_yint_planes")
    return y


def msd_steps(x, wp, scale, g, steps: int, mode: int = MODE_FP32) -> np.ndarray:
    """MSD with `steps` unfold steps (R16): y [M, N] float64."""
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_msd_steps(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g, mode, steps, _ptr(y)),
           "msd_steps")
    return y


def msd_at_steps(x, wp, scale, g, steps: int, rows, cols, mode: int = MODE_FP32) -> np.ndarray:
    """MSD with `steps` unfold steps at y[rows[i], cols[i]] only (float64)."""
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    order, r, c = _sorted_pairs(rows, cols)
    out = np.empty(r.size, np.float64)
    _check(_load().oracle_msd_at_steps(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g, mode, steps,
                                       _ptr(r), _ptr(c), r.size, _ptr(out)), "msd_at_steps")
    res = np.empty_like(out)
    res[order] = out
    return res


def _sorted_pairs(rows, cols):
    rows = np.asarray(rows, np.int32)
    cols = np.asarray(cols, np.int32)
    order = np.lexsort((cols, rows))
    return order, np.ascontiguousarray(rows[order]), np.ascontiguousarray(cols[order])


def msd_at(x, wp, scale, g, rows, cols, mode: int = MODE_FP32) -> np.ndarray:
    """MSD outputs y[rows[i], cols[i]] only (float64)."""
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    order, r, c = _sorted_pairs(rows, cols)
    out = np.empty(r.size, np.float64)
    _check(_load().oracle_msd_at(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g, mode,
                                 _ptr(r), _ptr(c), r.size, _ptr(out)), "msd_at")
    res = np.empty_like(out)
    res[order] = out
    return res


def dequant(x, wp, scale, g) -> np.ndarray:
    """Exact y = x . (scale (.) W) in float64: [M, N]."""
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_dequant(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g, _ptr(y)),
           "dequant")
    return y


def dequant_at(x, wp, scale, g, rows, cols) -> np.ndarray:
    x = _c(x, np.float16)
    wp = _c(wp, np.uint8)
    scale = _c(scale, np.float16)
    M, K = x.shape
    N = wp.shape[1]
    order, r, c = _sorted_pairs(rows, cols)
    out = np.empty(r.size, np.float64)
    _check(_load().oracle_dequant_at(_ptr(x), _ptr(wp), _ptr(scale), M, K, N, g,
                                     _ptr(r), _ptr(c), r.size, _ptr(out)), "dequant_at")
    res = np.empty_like(out)
    res[order] = out
    return res


def grouped(op: str, x, wps, scales, offsets, g) -> np.ndarray:
    """Per-expert oracle over contiguous token segments: y [T, N] float64.

    Expert e owns tokens offsets[e] .. offsets[e+1]-1 and uses wps[e], scales[e].
    """
    x = _c(x, np.float16)
    T = x.shape[0]
    N = wps[0].shape[1]
    y = np.zeros((T, N), np.float64)
    fn = msd if op == "msd" else dequant
    for e in range(len(wps)):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            y[a:b] = fn(x[a:b], wps[e], scales[e], g)
    return y


def grouped_at(op: str, x, wps, scales, offsets, g, rows, cols) -> np.ndarray:
    """Per-expert oracle at listed (token, column) pairs."""
    rows = np.asarray(rows, np.int64)
    cols = np.asarray(cols, np.int64)
    offsets = np.asarray(offsets, np.int64)
    out = np.empty(rows.size, np.float64)
    experts = np.searchsorted(offsets, rows, side="right") - 1
    fn = msd_at if op == "msd" else dequant_at
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        a, b = int(offsets[e]), int(offsets[e + 1])
        out[sel] = fn(x[a:b], wps[e], scales[e], g, rows[sel] - a, cols[sel])
    return out


def moe_align(topk_ids, E):
    """Stable grouping of the router's entries by expert (reading R13 of the C
    file): returns offsets [E+1], sorted_token [T*topk], inv_pos [T*topk] and
    the number of entries whose id lies outside [0, E)."""
    ids = _c(np.asarray(topk_ids, np.int32), np.int32)
    T, topk = ids.shape
    offsets = np.empty(E + 1, np.int32)
    st = np.empty(T * topk, np.int32)
    inv = np.empty(T * topk, np.int32)
    dropped = _load().oracle_moe_align(_ptr(ids), T, topk, E, _ptr(offsets), _ptr(st), _ptr(inv))
    if dropped < 0:
        raise ValueError("oracle moe_align failed")
    return offsets, st, inv, dropped


def moe_combine(y_sorted, inv_pos, weights):
    """Gate-weighted un-permute (reading R14): fp16 y_sorted [rows, N] -> fp16 y [T, N]."""
    ys = _c(np.asarray(y_sorted, np.float16), np.float16)
    inv = _c(np.asarray(inv_pos, np.int32), np.int32)
    w = _c(np.asarray(weights, np.float32), np.float32)
    T, topk = w.shape
    N = ys.shape[1]
    y = np.empty((T, N), np.uint16)
    _check(_load().oracle_moe_combine(_ptr(ys), _ptr(inv), _ptr(w), T, topk, N, _ptr(y)), "moe_combine")
    return y.view(np.float16)


def moe(op: str, x, topk_ids, weights, wps, scales, g) -> np.ndarray:
    """The routed grouped form end to end: y [T, N] float64.

    The entries are grouped by expert (moe_align), the per-expert matmul runs
    on the gathered rows (grouped), and token t's rows are added with its
    gate weights in binary64 (no binary16 rounding in between)."""
    x = _c(x, np.float16)
    w = np.asarray(weights, np.float64)
    T, topk = w.shape
    offsets, st, inv, _ = moe_align(topk_ids, len(wps))
    rows = int(offsets[-1])
    xs = x[st[:rows]] if rows else np.zeros((0, x.shape[1]), np.float16)
    ys = grouped(op, xs, wps, scales, offsets, g)
    y = np.zeros((T, ys.shape[1] if rows else wps[0].shape[1]), np.float64)
    for t in range(T):
        for j in range(topk):
            pos = int(inv[t * topk + j])
            if pos >= 0:
                y[t] += w[t, j] * ys[pos]
    return y


def bf16_to_double(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 values."""
    b = _c(np.asarray(b, dtype=np.uint16), np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().oracle_bf16s_to_double(_ptr(b), b.size, _ptr(out))
    return out


def dequant_bf16(x_bits, wp, scale_bits, g) -> np.ndarray:
    """Exact y = x . (scale (.) W) in float64 with bf16 x and scale given as
    uint16 bit patterns [M, K] / [K/g, N] (reading R15 of the C file)."""
    x = _c(np.asarray(x_bits, np.uint16), np.uint16)
    wp = _c(wp, np.uint8)
    sc = _c(np.asarray(scale_bits, np.uint16), np.uint16)
    M, K = x.shape
    N = wp.shape[1]
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_dequant_bf16(_ptr(x), _ptr(wp), _ptr(sc), M, K, N, g, _ptr(y)), "dequant_bf16")
    return y
