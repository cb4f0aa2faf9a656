"""GPU parity of the routing prep of the grouped form (router entries grouped
by expert, x gathered, y added back with the gate weights) against the CPU
oracle.  The grouping is unique (stable by entry), so it is compared bit for
bit; the end-to-end results use the MSD and dequant tolerances of the dense
tests."""
import numpy as np
import pytest

import oracle
from inputs import make_case
from test_gpu_parity import assert_deq_close, assert_msd_close, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import weight_only_int4_a16w4_b200 as w4
    return w4


def _ids(rng, T, topk, E, invalid=False):
    ids = rng.integers(0, E, (T, topk)).astype(np.int32)
    if invalid:
        ids[rng.random((T, topk)) < 0.05] = E + 3
        ids[0, 0] = -1
    return ids


def _align(w4, ids, E):
    import torch
    T, topk = ids.shape
    d_ids = torch.from_numpy(ids).cuda()
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    st = torch.full((T * topk,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((T * topk,), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    w4.w4a16_moe_align(d_ids, T, topk, E, offsets, st, inv, ws)
    return offsets.cpu().numpy(), st.cpu().numpy(), inv.cpu().numpy(), w4.w4a16_read_status(ws)


@pytest.mark.parametrize("T,topk,E,invalid", [
    (1, 1, 1, False),          # a single entry
    (37, 2, 5, False),         # ragged last batch of 32 entries
    (4096, 1, 8, False),       # the grouped workload's token count
    (1000, 8, 64, False),      # the most experts
    (333, 3, 16, True),        # ids outside [0, E) take no row
    (31, 4, 64, False),        # fewer entries than experts * warps
])
def test_moe_align_matches_oracle(w4, T, topk, E, invalid):
    rng = np.random.default_rng(T * 7 + topk * 3 + E)
    ids = _ids(rng, T, topk, E, invalid)
    off, st, inv, status = _align(w4, ids, E)
    r_off, r_st, r_inv, dropped = oracle.moe_align(ids, E)
    np.testing.assert_array_equal(off, r_off)
    np.testing.assert_array_equal(st, r_st)
    np.testing.assert_array_equal(inv, r_inv)
    assert status == (w4.DEVICE_BAD_EXPERT if dropped else 0)


def test_moe_gather_is_exact(w4):
    import torch
    rng = np.random.default_rng(3)
    T, topk, E, K = 300, 2, 7, 520
    ids = _ids(rng, T, topk, E, invalid=True)
    _, st, _, _ = oracle.moe_align(ids, E)
    x = rng.standard_normal((T, K)).astype(np.float16)
    xs = torch.full((T * topk, K), float("nan"), dtype=torch.float16, device="cuda")
    w4.w4a16_moe_gather(torch.from_numpy(x).cuda(), torch.from_numpy(st).cuda(), T * topk, K, xs)
    ref = np.zeros((T * topk, K), np.float16)
    ref[st >= 0] = x[st[st >= 0]]
    np.testing.assert_array_equal(xs.cpu().numpy().view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("T,topk,N", [(1, 1, 8), (200, 2, 264), (64, 8, 4096)])
def test_moe_combine_within_one_ulp(w4, T, topk, N):
    import torch
    rng = np.random.default_rng(T + topk + N)
    E = 6
    ids = _ids(rng, T, topk, E, invalid=True)
    _, _, inv, _ = oracle.moe_align(ids, E)
    ys = rng.standard_normal((T * topk, N)).astype(np.float16)
    w = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    y = torch.empty((T, N), dtype=torch.float16, device="cuda")
    w4.w4a16_moe_combine(torch.from_numpy(ys).cuda(), torch.from_numpy(inv).cuda(), torch.from_numpy(w).cuda(),
                         T, topk, N, y)
    got = y.cpu().numpy().astype(np.float64)
    ref = oracle.moe_combine(ys, inv, w).astype(np.float64)
    # fp32 sums vs binary64 sums, each rounded to fp16 once: one fp16 unit in
    # the last place at most
    ulp = np.spacing(np.maximum(np.abs(got), np.abs(ref)).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= ulp)


@pytest.mark.parametrize("op", ["msd", "dequant"])
@pytest.mark.parametrize("T,topk,E,K,N,g,invalid", [
    (37, 2, 5, 256, 264, 64, False),
    (150, 2, 8, 512, 136, 128, True),
    (9, 1, 3, 1024, 520, 256, False),
    (200, 1, 4, 256, 264, 64, True),       # one expert per token: fused un-permute, dropped ids give zero rows
    (300, 1, 8, 512, 136, 128, False),     # fused un-permute on the large tiles, ragged segments
])
def test_moe_matmul_end_to_end(w4, op, T, topk, E, K, N, g, invalid):
    import torch
    rng = np.random.default_rng(T * 11 + E)
    c = make_case(T, K, N, g, seed=T + K + N, E=E)
    ids = _ids(rng, T, topk, E, invalid)
    wts = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    dev = upload(w4, c)
    code = w4.OP_MSD if op == "msd" else w4.OP_DEQUANT
    ws = torch.zeros(w4.w4a16_moe_workspace_size(code, T, topk, K, N, g, E), dtype=torch.uint8, device="cuda")
    y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
    w4.w4a16_moe_matmul(code, dev["x"], torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(), dev["wp"],
                        dev["scale"], E, T, topk, K, N, g, y, ws)
    status = w4.w4a16_read_status(ws)
    assert status == (w4.DEVICE_BAD_EXPERT if invalid else 0)
    ref = oracle.moe(op, c.x, ids, wts, c.wp, c.scale, g)
    got = y.cpu().numpy().astype(np.float64)
    (assert_msd_close if op == "msd" else assert_deq_close)(got, ref, f"moe {op} {T}x{topk} E{E}")
