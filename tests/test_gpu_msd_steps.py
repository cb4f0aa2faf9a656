"""GPU parity of MSD with 2 and 4 unfold steps (reading R16 of the oracle)
against the oracle's S-step functions, through the C ABI.

Bars: the per-group int32 Y_1..Y_S and A_max from the debug window are
bit-exact against the oracle's S-step expansion and integer contraction
(both sides take the digit decisions in IEEE binary32); y meets the MSD bar
|y - y_oracle| <= 2e-3 * max|y_oracle| + 1e-3 against the oracle's S-step
binary64 result.  Every dispatch branch is covered: the warp-MMA GEMV
(S * M <= 8, g % 128 == 0), the tensor-core decode tile (M <= 16), the large
tile (64 tokens for S = 2, 32 for S = 4) and the grouped form.
"""
import numpy as np
import pytest

import oracle
from inputs import make_case, make_workload
from test_gpu_parity import assert_msd_close, upload

pytestmark = pytest.mark.gpu

OPS = {2: 3, 3: 0, 4: 4}      # steps -> W4A16_OP_* code


def _t():
    import torch
    return torch


def run_steps(w4, S, c, dev):
    torch = _t()
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.float16, device="cuda")
    ws = w4.alloc_workspace(OPS[S], c.M, c.K, c.N, c.g)
    w4.w4a16_msd_matmul_steps(S, dev["x"], dev["wp"][0], dev["scale"][0], c.M, c.K, c.N, c.g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    return y.cpu().numpy().astype(np.float64)


def check_yint_steps(w4, S, c, dev, m0, m1, n0, n1):
    torch = _t()
    G = c.K // c.g
    yint = torch.full((S, m1 - m0, G, n1 - n0), -12345, dtype=torch.int32, device="cuda")
    amax = torch.full((m1 - m0, G), -1.0, dtype=torch.float32, device="cuda")
    ws = w4.alloc_workspace(OPS[S], c.M, c.K, c.N, c.g)
    w4.w4a16_msd_debug_yint_steps(S, dev["x"], dev["wp"][0], c.M, c.K, c.N, c.g, m0, m1, n0, n1, yint, amax, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    ref_amax, a = oracle.msd_expand_steps(c.x[m0:m1], c.g, S)
    ref = oracle.msd_yint_planes(a, np.ascontiguousarray(c.wp[0][:, n0:n1]), n1 - n0, c.g)
    assert np.array_equal(amax.cpu().numpy().astype(np.float64), ref_amax), "A_max differs"
    got = yint.cpu().numpy().astype(np.int64)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"S={S}: {len(bad)} Y_int mismatches, first at {bad[0]}"


SHAPES = [
    # (M, K, N, g)                 branch for S = 2 / S = 4
    (1, 512, 264, 128),            # warp-MMA GEMV / warp-MMA GEMV
    (2, 1024, 136, 256),           # warp-MMA GEMV, groups over two chunks / warp-MMA GEMV
    (3, 512, 128, 128),            # warp-MMA GEMV (3 tokens x 2 planes) / decode tile
    (4, 384, 256, 128),            # warp-MMA GEMV (all 8 rows) / decode tile
    (5, 256, 256, 64),             # decode tile, g = 64
    (16, 256, 264, 32),            # decode tile, split-K, four groups per chunk
    (17, 512, 136, 128),           # large tile, one token past the decode tile
    (70, 384, 256, 64),            # large tile, ragged token tail
    (130, 256, 520, 128),          # large tile, ragged in every dimension
]


@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("M,K,N,g", SHAPES)
def test_msd_steps_match_oracle(cuda_lib, S, M, K, N, g):
    w4 = cuda_lib
    c = make_case(M, K, N, g, seed=M * 100 + K + N + g + S)
    if M > 2:
        c.x[1, :g] = 0                      # an all-zero group
    dev = upload(w4, c)
    y = run_steps(w4, S, c, dev)
    assert_msd_close(y, oracle.msd_steps(c.x, c.wp[0], c.scale[0], g, S), f"S={S} {M}x{K}x{N} g{g}")
    check_yint_steps(w4, S, c, dev, 0, M, 0, N)


def test_three_steps_is_the_plain_msd_call(cuda_lib):
    """steps = 3 runs the same kernels as w4a16_msd_matmul: identical bits."""
    w4 = cuda_lib
    torch = _t()
    for M in (1, 16, 70):
        c = make_case(M, 512, 264, 128, seed=900 + M)
        dev = upload(w4, c)
        y3 = run_steps(w4, 3, c, dev)
        y = torch.empty((M, c.N), dtype=torch.float16, device="cuda")
        ws = w4.alloc_workspace(w4.OP_MSD, M, c.K, c.N, c.g)
        w4.w4a16_msd_matmul(dev["x"], dev["wp"][0], dev["scale"][0], M, c.K, c.N, c.g, y, ws)
        assert np.array_equal(y.cpu().numpy().astype(np.float64), y3)


def test_more_steps_are_closer_to_the_exact_product(cuda_lib):
    """The accuracy side of the knob, on the GPU's own results: the error
    against the exact dequant product shrinks from 2 to 3 to 4 steps."""
    w4 = cuda_lib
    c = make_case(32, 1024, 512, 128, seed=4242, outliers=False)
    dev = upload(w4, c)
    exact = oracle.dequant(c.x, c.wp[0], c.scale[0], c.g)
    errs = [np.sqrt(np.mean((run_steps(w4, S, c, dev) - exact) ** 2)) for S in (2, 3, 4)]
    assert errs[0] > errs[1] > errs[2], errs


@pytest.mark.parametrize("S", [2, 4])
def test_grouped_msd_steps(cuda_lib, S):
    w4 = cuda_lib
    torch = _t()
    T, K, N, g, E = 150, 256, 264, 64, 4
    c = make_case(T, K, N, g, seed=77 + S, E=E)
    dev = upload(w4, c)
    y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
    ws = w4.alloc_workspace(OPS[S], T, K, N, g, E=E)
    w4.w4a16_grouped_matmul(OPS[S], dev["x"], dev["wp"], dev["scale"], dev["offsets"], E, T, K, N, g, y, ws)
    torch.cuda.synchronize()
    assert w4.w4a16_read_status(ws) == 0
    ref = np.zeros((T, N))
    for e in range(E):
        r0, r1 = int(c.offsets[e]), int(c.offsets[e + 1])
        if r1 > r0:
            ref[r0:r1] = oracle.msd_steps(c.x[r0:r1], c.wp[e], c.scale[e], g, S)
    assert_msd_close(y.cpu().numpy().astype(np.float64), ref, f"grouped S={S}")


@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("name", ["decode_m1", "decode_m16", "prefill"])
def test_workload_msd_steps_sampled(cuda_lib, S, name):
    """The full-size workloads with 2 and 4 steps: 1024 sampled outputs and a
    Y_int window at the ragged end."""
    w4 = cuda_lib
    c = make_workload(name)
    dev = upload(w4, c)
    y = run_steps(w4, S, c, dev)
    rng = np.random.default_rng(S * 10 + len(name))
    rows, cols = rng.integers(0, c.M, 1024), rng.integers(0, c.N, 1024)
    assert_msd_close(y[rows, cols], oracle.msd_at_steps(c.x, c.wp[0], c.scale[0], c.g, S, rows, cols),
                     f"{name} S={S}")
    m0 = max(0, c.M - 16)
    check_yint_steps(w4, S, c, dev, m0, c.M, c.N - 40, c.N)


@pytest.mark.parametrize("S,topk", [(2, 1), (4, 2)])
def test_routed_msd_steps(cuda_lib, S, topk):
    """The routed form (grouping, gather, grouped matmul, un-permute) with the
    step variants: per token the gate-weighted sum over its experts of the
    oracle's S-step rows."""
    w4 = cuda_lib
    torch = _t()
    T, E, K, N, g = 45, 3, 256, 136, 64
    rng = np.random.default_rng(100 + S)
    c = make_case(T, K, N, g, seed=300 + S, E=E, grouped=False)
    ids = rng.integers(0, E, (T, topk)).astype(np.int32)
    wts = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    dev = upload(w4, c)
    ws = torch.zeros(w4.w4a16_moe_workspace_size(OPS[S], T, topk, K, N, g, E), dtype=torch.uint8, device="cuda")
    y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
    w4.w4a16_moe_matmul(OPS[S], dev["x"], torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(), dev["wp"],
                        dev["scale"], E, T, topk, K, N, g, y, ws)
    assert w4.w4a16_read_status(ws) == 0
    rows = [oracle.msd_steps(c.x, c.wp[e], c.scale[e], g, S) for e in range(E)]
    ref = np.zeros((T, N))
    for t in range(T):
        for j in range(topk):
            ref[t] += float(wts[t, j]) * rows[int(ids[t, j])][t]
    assert_msd_close(y.cpu().numpy().astype(np.float64), ref, f"routed S={S} topk={topk}")
