"""GPU parity of the dequant variant with bf16 activations (bf16 x, scale
and y; the INT4 + BF16 pairing of the Humming article) against the oracle's
exact binary64 y, through the C ABI.

Bar (reading R15 of the oracle, derived from the arithmetic): the library
computes y in fp32 from exact bf16 products and rounds it to bf16 once, so
per element

    |y_gpu - y| <= u * (|y| + c*S) + c*S,        u = 2^-8 (bf16 unit roundoff),

with S = sum_k |x_k| * |scale_k * w_k| and c = (g/16 + K/g + 24) * 2^-23 the
fp32 budget: at most g/16 MMA steps inside a group, one scale multiply and
one add per group, and at most 24 further adds (warp or split-K partials),
each off by at most 2^-23 of a partial sum that S bounds.  A dropped piece,
a wrong scale or a transposed operand moves y by far more than this.
Full-size workloads are checked on a block of rows x columns that the oracle
computes whole.
"""
import numpy as np
import pytest

import oracle
from inputs import make_case, make_workload

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8


def fp32_budget(K, g):
    return (g / 16 + K / g + 24) * 2.0 ** -23


def _t():
    import torch
    return torch


def _dev_bf16(bits):
    torch = _t()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def upload(w4, c):
    torch = _t()
    dev = {"x": _dev_bf16(c.x)}
    dev["wp"] = [w4.repack(torch.from_numpy(wp).cuda(), c.K, c.N) for wp in c.wp]
    dev["scale"] = [_dev_bf16(s) for s in c.scale]
    if c.offsets is not None:
        dev["offsets"] = torch.from_numpy(c.offsets).cuda()
    return dev


def run_dense(w4, c, dev):
    torch = _t()
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = w4.alloc_workspace(w4.OP_DEQUANT_BF16, c.M, c.K, c.N, c.g)
    w4.w4a16_dequant_matmul_bf16(dev["x"], dev["wp"][0], dev["scale"][0], c.M, c.K, c.N, c.g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.float().cpu().numpy().astype(np.float64)


def run_grouped(w4, c, dev):
    torch = _t()
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = w4.alloc_workspace(w4.OP_DEQUANT_BF16, c.M, c.K, c.N, c.g, E=c.E)
    w4.w4a16_grouped_matmul(w4.OP_DEQUANT_BF16, dev["x"], dev["wp"], dev["scale"], dev["offsets"], c.E, c.M,
                            c.K, c.N, c.g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.float().cpu().numpy().astype(np.float64)


def magnitude(xb, wp, sb, g):
    """S = |x| . |scale (.) W| in float64 (the rounding budget's scale)."""
    K, N = xb.shape[1], wp.shape[1]
    x = np.abs(oracle.bf16_to_double(xb))
    s = np.abs(oracle.bf16_to_double(sb))
    w = np.abs(oracle.unpack_w(np.ascontiguousarray(wp), K, N).astype(np.float64))
    return x @ (np.repeat(s, g, axis=0) * w)


def assert_bf16_close(y, ref, S, K, g, what=""):
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    c = fp32_budget(K, g)
    tol = U_BF16 * (np.abs(ref) + c * S) + c * S
    err = np.abs(y - ref)
    i = np.unravel_index(np.argmax(err / tol), err.shape)
    assert np.all(err <= tol), f"{what}: err {err[i]:.3e} > tol {tol[i]:.3e} at {i} (gpu {y[i]}, oracle {ref[i]})"


def check_dense_block(c, y, rows, cols, what):
    xb = c.x[rows]
    wp = np.ascontiguousarray(c.wp[0][:, cols])
    sb = np.ascontiguousarray(c.scale[0][:, cols])
    ref = oracle.dequant_bf16(xb, wp, sb, c.g)
    assert_bf16_close(y[np.ix_(rows, cols)], ref, magnitude(xb, wp, sb, c.g), c.K, c.g, what)


# ---------------------------------------------------------------- small shapes, full comparison

SMALL = [
    # (M, K, N, g)                       what it covers
    (16, 256, 256, 64),                  # decode tile, split-K over groups of 64
    (1, 256, 128, 128),                  # one row: warp-MMA GEMV
    (5, 384, 136, 64),                   # ragged N, g = 64 (decode tile: no CUDA-core GEMV for bf16)
    (16, 192, 256, 64),                  # K not a multiple of 128
    (3, 512, 256, 256),                  # group spanning two K chunks (warp-MMA GEMV)
    (9, 512, 384, 32),                   # four groups per K chunk
    (17, 256, 264, 128),                 # first M above the decode tile
    (70, 512, 256, 64),                  # several token tiles, ragged tail, one MMA issuer
    (130, 384, 520, 128),                # ragged in every dimension, two MMA issuers
    (8, 1024, 264, 128),                 # the largest warp-MMA GEMV row count
    (2, 4096, 1032, 128),                # a long K with ragged column blocks
    (1, 1024, 8200, 128),                # the 32-warp GEMV instance (M <= 2, N >= 8192)
]


@pytest.mark.parametrize("M,K,N,g", SMALL)
def test_dense_bf16_matches_oracle(cuda_lib, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 1000 + K + N + g, act="bf16")
    dev = upload(w4, c)
    y = run_dense(w4, c, dev)
    ref = oracle.dequant_bf16(c.x, c.wp[0], c.scale[0], g)
    assert_bf16_close(y, ref, magnitude(c.x, c.wp[0], c.scale[0], g), K, g, f"bf16 {M}x{K}x{N} g{g}")


def test_dense_bf16_degenerate(cuda_lib):
    """All-zero x gives exact zeros; a single non-zero entry gives one scaled
    weight row, exact in bf16 when the scale is a power of two."""
    w4 = cuda_lib
    torch = _t()
    c = make_case(3, 256, 136, 64, seed=77, act="bf16")
    c.x[:] = 0
    dev = upload(w4, c)
    assert np.all(run_dense(w4, c, dev) == 0.0)
    c.x[1, 70] = 0x4000                      # 2.0
    c.scale[0][:] = 0x3E80                   # 0.25
    dev = upload(w4, c)
    y = run_dense(w4, c, dev)
    w = oracle.unpack_w(c.wp[0], c.K, c.N).astype(np.float64)
    assert np.array_equal(y[1], 0.5 * w[70])
    assert np.all(y[[0, 2]] == 0.0)
    del torch


def test_dense_bf16_m0_is_noop(cuda_lib):
    w4 = cuda_lib
    w4.w4a16_dequant_matmul_bf16(None, None, None, 0, 256, 256, 64, None, None, 0)


# ---------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("name,nrows", [("decode_m1", 1), ("decode_m16", 16), ("prefill", 24)])
def test_workload_bf16_block(cuda_lib, name, nrows):
    """The decode and prefill workloads in bf16, launched as the benchmark
    launches them; a block of rows x 320 columns (random plus the last 64)
    checked against the oracle."""
    w4 = cuda_lib
    c = make_workload(name, act="bf16")
    dev = upload(w4, c)
    y = run_dense(w4, c, dev)
    rng = np.random.default_rng(len(name))
    rows = np.sort(rng.choice(c.M, size=min(nrows, c.M), replace=False))
    if c.M > nrows:
        rows[-1] = c.M - 1
    cols = np.concatenate([np.sort(rng.choice(c.N - 64, 256, replace=False)), np.arange(c.N - 64, c.N)])
    check_dense_block(c, y, rows, cols, f"bf16 {name}")


# ---------------------------------------------------------------- grouped and routed forms

def _grouped_ref(c):
    T = c.M
    ref = np.zeros((T, c.N))
    S = np.zeros((T, c.N))
    for e in range(c.E):
        r0, r1 = int(c.offsets[e]), int(c.offsets[e + 1])
        if r1 > r0:
            ref[r0:r1] = oracle.dequant_bf16(c.x[r0:r1], c.wp[e], c.scale[e], c.g)
            S[r0:r1] = magnitude(c.x[r0:r1], c.wp[e], c.scale[e], c.g)
    return ref, S


@pytest.mark.parametrize("T,K,N,g,E", [
    (70, 256, 264, 64, 3),               # ragged experts, one MMA issuer
    (300, 512, 136, 128, 5),             # two MMA issuers
    (9, 256, 128, 128, 4),               # fewer tokens than a tile, empty experts likely
])
def test_grouped_bf16_matches_oracle(cuda_lib, T, K, N, g, E):
    w4 = cuda_lib
    c = make_case(T, K, N, g, seed=T + K + N + E, E=E, act="bf16")
    dev = upload(w4, c)
    ref, S = _grouped_ref(c)
    assert_bf16_close(run_grouped(w4, c, dev), ref, S, K, g, f"grouped bf16 T{T} E{E}")


@pytest.mark.parametrize("topk", [1, 2])
def test_moe_matmul_bf16_end_to_end(cuda_lib, topk):
    """Router entries grouped, gathered, multiplied and added back with the
    gate weights, all in bf16: each row's y is rounded to bf16 once before the
    fp32 gate-weighted sum (topk = 1: the weight is applied in the matmul's
    stores, one rounding), so the bar adds u times the rows' weighted sizes."""
    w4 = cuda_lib
    torch = _t()
    T, E, K, N, g = 37, 5, 256, 136, 64
    rng = np.random.default_rng(5)
    c = make_case(T, K, N, g, seed=91, E=E, grouped=False, act="bf16")
    ids = rng.integers(0, E, (T, topk)).astype(np.int32)
    wts = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    dev = upload(w4, c)
    ws = torch.zeros(w4.w4a16_moe_workspace_size(w4.OP_DEQUANT_BF16, T, topk, K, N, g, E), dtype=torch.uint8,
                     device="cuda")
    y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    w4.w4a16_moe_matmul(w4.OP_DEQUANT_BF16, dev["x"], torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(),
                        dev["wp"], dev["scale"], E, T, topk, K, N, g, y, ws)
    assert w4.w4a16_read_status(ws) == 0
    got = y.float().cpu().numpy().astype(np.float64)
    rows = {e: oracle.dequant_bf16(c.x, c.wp[e], c.scale[e], g) for e in range(E)}
    mags = {e: magnitude(c.x, c.wp[e], c.scale[e], g) for e in range(E)}
    ref = np.zeros((T, N))
    spread = np.zeros((T, N))
    budget = np.zeros((T, N))
    cb = fp32_budget(K, g)
    for t in range(T):
        for j in range(topk):
            e, wj = int(ids[t, j]), float(wts[t, j])
            ref[t] += wj * rows[e][t]
            spread[t] += wj * (np.abs(rows[e][t]) + cb * mags[e][t])
            budget[t] += wj * cb * mags[e][t]
    tol = U_BF16 * (np.abs(ref) + 2 * spread) + budget + 2.0 ** -22 * spread
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    i = np.unravel_index(np.argmax(err / tol), err.shape)
    assert np.all(err <= tol), f"moe bf16: err {err[i]:.3e} > tol {tol[i]:.3e} at {i}"
