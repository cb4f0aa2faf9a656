"""Pins for the CPU oracle: each test ties the oracle to something other than
itself -- the binary16 format via numpy's converters, hand-worked values,
invariants the method guarantees, the truncation bound against an exact
GEMM computed by numpy, integer brute force -- so that a dropped term, a
wrong sign, index or transposed operand in the oracle fails one of them.

Method source: "WeightQuantBatchMatmulExperiment 算子深度解析"
(bjdmk.com.cn/news/4847346), section 4.1, equations 1-11.
"""
import json
import os

import numpy as np
import pytest

import oracle
from inputs import make_case, pack_int4, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# 0.5 / (7.49 * 14.98^2): the largest value the dropped fourth digit can
# carry, relative to A_max, after three residual steps (eq. 2-7).
TRUNC = 0.5 / (7.49 * 14.98 * 14.98)


# ---------------------------------------------------------------- binary16

def test_half_to_double_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    ours = oracle.half_to_double(h)
    ref = h.astype(np.float64)
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    inf = np.isinf(ref)
    assert np.array_equal(ours[inf], ref[inf])


def test_double_to_half_matches_numpy_rounding():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        # exact ties between neighbouring halves, both parities
        (np.arange(4096, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        np.array([65504.0, 65519.99, 65520.0, 1e6, -0.0, 0.0, 6e-8, 2.9e-8, 3.0e-8]),
    ])
    ours = oracle.double_to_half(v).view(np.uint16)
    ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------- int4 decode

def test_unpack_nibble_order_and_sign_literal():
    # byte 0x9F: low nibble 0xF -> W[0] = -1, high nibble 0x9 -> W[1] = -7
    # byte 0x70: low 0x0 -> 0, high 0x7 -> 7 ; byte 0x08: low 0x8 -> -8, high 0
    wp = np.array([[0x9F, 0x70, 0x08]], dtype=np.uint8)
    w = oracle.unpack_w(wp, 2, 3)
    assert w.tolist() == [[-1, 0, -8], [-7, 7, 0]]


def test_unpack_every_byte():
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    w = oracle.unpack_w(b, 2, 256)
    lo = np.arange(256) & 15
    hi = np.arange(256) >> 4
    assert np.array_equal(w[0], np.where(lo >= 8, lo - 16, lo))
    assert np.array_equal(w[1], np.where(hi >= 8, hi - 16, hi))


# ---------------------------------------------------------------- worked example

def _golden():
    with open(os.path.join(GOLDEN, "msd_worked_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_worked_example_digits_and_yint(mode):
    ex = _golden()
    g = ex["g"]
    x = np.array([ex["x"]], dtype=np.float16)
    w = np.array(ex["w"], dtype=np.int8)
    amax, a = oracle.msd_expand(x, g, mode)
    assert amax[0, 0] == ex["amax"]
    assert a[0, 0].tolist() == ex["A1"]
    assert a[1, 0].tolist() == ex["A2"]
    assert a[2, 0].tolist() == ex["A3"]
    yint = oracle.msd_yint(a, pack_int4(w), w.shape[1], g)
    assert yint[0, 0, 0].tolist() == ex["Y1"]
    assert yint[1, 0, 0].tolist() == ex["Y2"]
    assert yint[2, 0, 0].tolist() == ex["Y3"]


def test_worked_example_output():
    ex = _golden()
    g = ex["g"]
    x = np.array([ex["x"]], dtype=np.float16)
    w = np.array(ex["w"], dtype=np.int8)
    scale = np.array([ex["scale"]], dtype=np.float16)
    y = oracle.msd(x, pack_int4(w), scale, g)
    np.testing.assert_allclose(y[0], ex["y_msd"], rtol=1e-12, atol=0)
    ye = oracle.dequant(x, pack_int4(w), scale, g)
    np.testing.assert_allclose(ye[0], ex["y_exact"], rtol=1e-15, atol=0)
    assert np.all(np.abs(y[0] - ye[0]) <= np.array(ex["truncation_bound"]))


# ---------------------------------------------------------------- invariants

def _adversarial_x(rng, M, K, g):
    x = rng.standard_normal((M, K)).astype(np.float16)
    x[0] = 0                                  # all-zero groups
    x[1, :g] = np.float16(3.0)                # all entries equal +A_max
    x[1, g:2 * g] = np.float16(-0.5)          # all entries equal -A_max
    x[2] = rng.integers(-3, 4, K).astype(np.float16)     # small integers
    x[3] *= np.float16(1e-4)                  # tiny values (subnormals)
    x[4, ::7] *= np.float16(2000)             # big outliers
    return x


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_digits_bounded_by_seven(mode):
    """|tmp1| <= 7.49 and each residual |tmp - round(tmp)| <= 0.5, so after the
    x14.98 rescale every digit satisfies |A_i| <= 7 (fits symmetric int4)."""
    rng = np.random.default_rng(7)
    for g in (32, 64, 128):
        x = _adversarial_x(rng, 8, 512, g)
        _, a = oracle.msd_expand(x, g, mode)
        assert np.abs(a).max() <= 7


def test_equal_magnitude_group_digits():
    """x = +-A_max everywhere: tmp1 = +-7.49 -> A1 = +-7; tmp2 = +-0.49*14.98 =
    +-7.3402 -> A2 = +-7; tmp3 = +-0.3402*14.98 = +-5.0962 -> A3 = +-5."""
    x = np.array([[2.0] * 4 + [-2.0] * 4], dtype=np.float16)
    amax, a = oracle.msd_expand(x, 4)
    assert amax.tolist() == [[2.0, 2.0]]
    assert a[:, 0, :4].tolist() == [[7] * 4, [7] * 4, [5] * 4]
    assert a[:, 0, 4:].tolist() == [[-7] * 4, [-7] * 4, [-5] * 4]


def test_zero_group_contributes_nothing():
    c = make_case(4, 256, 64, 64, seed=3)
    c.x[1, 64:128] = 0
    amax, a = oracle.msd_expand(c.x, 64)
    assert amax[1, 1] == 0 and not a[:, 1, 64:128].any()
    y = oracle.msd(c.x, c.wp[0], c.scale[0], 64)
    # zeroing the group's scale changes nothing for row 1
    s2 = c.scale[0].copy()
    s2[1] = 0
    y2 = oracle.msd(c.x, c.wp[0], s2, 64)
    assert np.array_equal(y[1], y2[1])
    assert not np.array_equal(y[0], y2[0])


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_digit_reconstruction(mode):
    """7.49*x/A_max = A1 + A2/14.98 + A3/14.98^2 + r/14.98^2 with |r| <= 0.5."""
    rng = np.random.default_rng(11)
    g = 64
    x = _adversarial_x(rng, 8, 256, g)
    amax, a = oracle.msd_expand(x, g, mode)
    xd = x.astype(np.float64)
    am = np.repeat(amax, g, axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = np.where(am > 0, 7.49 * xd / am, 0.0)
    rec = a[0] + a[1] / 14.98 + a[2] / 14.98 ** 2
    slack = 0.5 / 14.98 ** 2 * (1.0 if mode == oracle.MODE_FP64 else 1.02)
    assert np.abs(t - rec).max() <= slack + 1e-12


# ---------------------------------------------------------------- against exact GEMMs

def _exact_gemm(x, w, scale, g):
    """fp64 GEMM by numpy (a library primitive, another summation order)."""
    s = np.repeat(scale.astype(np.float64), g, axis=0)
    return x.astype(np.float64) @ (s * w.astype(np.float64))


def _truncation_bound(amax, w, scale, g):
    K, N = w.shape
    G = K // g
    absw = np.abs(w.astype(np.float64)).reshape(G, g, N).sum(axis=1)      # [G, N]
    return TRUNC * (amax @ (np.abs(scale.astype(np.float64)) * absw))     # [M, N]


@pytest.mark.parametrize("g", [32, 64, 128])
def test_dequant_oracle_matches_numpy_gemm(g):
    c = make_case(5, 512, 96, g, seed=20 + g, keep_w=True)
    y = oracle.dequant(c.x, c.wp[0], c.scale[0], g)
    ref = _exact_gemm(c.x, c.w[0], c.scale[0], g)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_dequant_integer_special_case_is_exact():
    """scale = 1 and small-integer x: the exact GEMM is an integer GEMM."""
    rng = np.random.default_rng(5)
    K, N, g = 256, 40, 64
    xi = rng.integers(-4, 5, (3, K))
    w = rng.integers(-8, 8, (K, N)).astype(np.int8)
    y = oracle.dequant(xi.astype(np.float16), pack_int4(w), np.ones((K // g, N), np.float16), g)
    assert np.array_equal(y, (xi @ w.astype(np.int64)).astype(np.float64))


def test_dequant_single_group_dot_product():
    """g = K, M = 1: one scale per column, a textbook dot product."""
    rng = np.random.default_rng(9)
    K, N = 64, 3
    x = rng.standard_normal((1, K)).astype(np.float16)
    w = rng.integers(-8, 8, (K, N)).astype(np.int8)
    s = np.array([[0.5, -0.25, 0.125]], np.float16)
    y = oracle.dequant(x, pack_int4(w), s, K)
    for n in range(N):
        ref = float(s[0, n]) * sum(float(x[0, k]) * int(w[k, n]) for k in range(K))
        assert abs(y[0, n] - ref) <= 1e-12 * max(1.0, abs(ref))


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
@pytest.mark.parametrize("g", [32, 64, 128])
def test_msd_within_truncation_bound_of_exact(mode, g):
    """The MSD result stays within the decomposition's truncation error of the
    exact GEMM (binary64 expansion: exactly; binary32: a 2% slack covers the
    gap between 7.49f/14.98f and 7.49/14.98 and the rounding of tmp)."""
    c = make_case(6, 512, 80, g, seed=40 + g, keep_w=True)
    c.x[2, :g] = 0
    amax, _ = oracle.msd_expand(c.x, g, mode)
    y = oracle.msd(c.x, c.wp[0], c.scale[0], g, mode)
    ye = _exact_gemm(c.x, c.w[0], c.scale[0], g)
    bound = _truncation_bound(amax, c.w[0], c.scale[0], g)
    slack = 1.0 if mode == oracle.MODE_FP64 else 1.02
    assert np.all(np.abs(y - ye) <= bound * slack + 1e-12)
    # and the error is not trivially zero: MSD is an approximation
    assert np.abs(y - ye).max() > 0


def test_msd_yint_matches_integer_gemm():
    c = make_case(4, 256, 48, 64, seed=77, keep_w=True)
    amax, a = oracle.msd_expand(c.x, 64)
    yint = oracle.msd_yint(a, c.wp[0], 48, 64)
    w = c.w[0].astype(np.int64)
    for r in range(3):
        for gi in range(4):
            ref = a[r].astype(np.int64)[:, gi * 64:(gi + 1) * 64] @ w[gi * 64:(gi + 1) * 64]
            assert np.array_equal(yint[r, :, gi], ref)
    # the magnitude bound |Y| <= 7 * 8 * g
    assert np.abs(yint).max() <= 7 * 8 * 64


def test_msd_brute_force_tiny():
    """Tiny shapes, every weight value: the stored-Y path (eq. 9 then 10-11)
    equals the fused per-row path, and both meet the truncation bound."""
    for K, g in ((2, 2), (4, 2), (8, 4), (8, 8)):
        for N in (1, 3):
            for seed in range(4):
                c = make_case(2, K, N, g, seed=1000 + seed, keep_w=True)
                amax, a = oracle.msd_expand(c.x, g)
                yint = oracle.msd_yint(a, c.wp[0], N, g)
                y1 = oracle.msd_combine(yint, amax, c.scale[0], K, g)
                y2 = oracle.msd(c.x, c.wp[0], c.scale[0], g)
                assert np.array_equal(y1, y2)
                ye = _exact_gemm(c.x, c.w[0], c.scale[0], g)
                bound = _truncation_bound(amax, c.w[0], c.scale[0], g)
                assert np.all(np.abs(y2 - ye) <= bound * 1.02 + 1e-15)
    # all 16 weight values in one column
    w = np.arange(-8, 8, dtype=np.int8).reshape(16, 1)
    x = np.linspace(-1, 1, 16).astype(np.float16).reshape(1, 16)
    s = np.array([[0.75]], np.float16)
    y = oracle.msd(x, pack_int4(w), s, 16)
    amax, a = oracle.msd_expand(x, 16)
    ye = _exact_gemm(x, w, s, 16)
    assert abs(y[0, 0] - ye[0, 0]) <= _truncation_bound(amax, w, s, 16)[0, 0] * 1.02


def test_sampled_outputs_match_full():
    c = make_case(7, 256, 64, 64, seed=5)
    rows = np.array([6, 0, 3, 3, 6, 1])
    cols = np.array([63, 0, 17, 2, 5, 40])
    y = oracle.msd(c.x, c.wp[0], c.scale[0], 64)
    assert np.array_equal(oracle.msd_at(c.x, c.wp[0], c.scale[0], 64, rows, cols), y[rows, cols])
    yd = oracle.dequant(c.x, c.wp[0], c.scale[0], 64)
    assert np.array_equal(oracle.dequant_at(c.x, c.wp[0], c.scale[0], 64, rows, cols),
                          yd[rows, cols])


def test_grouped_oracle_segments():
    c = make_case(40, 128, 32, 64, seed=9, E=3)
    c.offsets[:] = [0, 10, 10, 40]          # an empty expert in the middle
    y = oracle.grouped("dequant", c.x, c.wp, c.scale, c.offsets, 64)
    assert np.array_equal(y[:10], oracle.dequant(c.x[:10], c.wp[0], c.scale[0], 64))
    assert np.array_equal(y[10:], oracle.dequant(c.x[10:], c.wp[2], c.scale[2], 64))
    rows, cols = np.array([0, 9, 10, 39]), np.array([1, 2, 3, 31])
    assert np.array_equal(oracle.grouped_at("msd", c.x, c.wp, c.scale, c.offsets, 64, rows, cols),
                          oracle.grouped("msd", c.x, c.wp, c.scale, c.offsets, 64)[rows, cols])


def test_workload_table():
    """The five workloads keep the shapes the benchmark and parity tests use."""
    assert (workload(0).M, workload(0).K, workload(0).N, workload(0).g) == (16, 256, 256, 64)
    assert (workload(1).M, workload(1).K, workload(1).N, workload(1).g) == (1, 4096, 4096, 128)
    assert (workload(2).M, workload(2).N) == (16, 14336)
    assert (workload(3).M, workload(3).N) == (4096, 4096)
    assert (workload(4).E, workload(4).M, workload(4).N) == (8, 4096, 14336)


# ---------------------------------------------------------------- routing prep of the grouped form

def _numpy_grouping(ids, E):
    """Independent reference: numpy's stable argsort of the expert ids (ids
    outside [0, E) sort last and take no row)."""
    flat = ids.reshape(-1).astype(np.int64)
    key = np.where((flat >= 0) & (flat < E), flat, E)
    order = np.argsort(key, kind="stable")
    valid = int(np.sum(key < E))
    counts = np.bincount(key, minlength=E + 1)[:E]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sorted_token = np.full(flat.size, -1, np.int32)
    sorted_token[:valid] = order[:valid] // ids.shape[1]
    inv = np.full(flat.size, -1, np.int32)
    inv[order[:valid]] = np.arange(valid)
    return offsets, sorted_token, inv, flat.size - valid


@pytest.mark.parametrize("T,topk,E,lo", [(1, 1, 1, 0), (37, 2, 8, -1), (256, 8, 64, 0), (500, 3, 5, -2)])
def test_moe_align_is_a_stable_grouping(T, topk, E, lo):
    rng = np.random.default_rng(T * 31 + topk)
    ids = rng.integers(lo, E + 1, (T, topk)).astype(np.int32)      # includes invalid ids when lo < 0 or = E
    got = oracle.moe_align(ids, E)
    ref = _numpy_grouping(ids, E)
    for a, b in zip(got[:3], ref[:3]):
        np.testing.assert_array_equal(a, b)
    assert got[3] == ref[3]


def test_moe_combine_topk1_unit_weight_is_the_permutation():
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 4, (50, 1)).astype(np.int32)
    _, _, inv, _ = oracle.moe_align(ids, 4)
    ys = rng.standard_normal((50, 24)).astype(np.float16)
    y = oracle.moe_combine(ys, inv, np.ones((50, 1), np.float32))
    np.testing.assert_array_equal(y.view(np.uint16), ys[inv].view(np.uint16))


def test_moe_combine_is_linear_in_the_gate_weights():
    """A one-hot weight picks one slot's row exactly; doubling every weight
    doubles the result exactly (a power-of-two scale commutes with rounding)."""
    rng = np.random.default_rng(6)
    T, topk, E, N = 40, 3, 6, 16
    ids = rng.integers(0, E, (T, topk)).astype(np.int32)
    _, _, inv, _ = oracle.moe_align(ids, E)
    ys = (rng.standard_normal((T * topk, N)) * 0.25).astype(np.float16)
    for j in range(topk):
        w = np.zeros((T, topk), np.float32)
        w[:, j] = 1
        np.testing.assert_array_equal(oracle.moe_combine(ys, inv, w).view(np.uint16),
                                      ys[inv.reshape(T, topk)[:, j]].view(np.uint16))
    w = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    a = oracle.moe_combine(ys, inv, w).astype(np.float64)
    b = oracle.moe_combine(ys, inv, 2 * w).astype(np.float64)
    np.testing.assert_array_equal(2 * a, b)


def test_moe_pipeline_matches_per_token_experts():
    """The routed pipeline equals, token by token, the gate-weighted sum of
    the token's own experts' dequant products (no permutation involved)."""
    rng = np.random.default_rng(7)
    T, topk, E, K, N, g = 9, 2, 3, 64, 16, 32
    c = make_case(T, K, N, g, seed=11, E=E)
    ids = rng.integers(-1, E, (T, topk)).astype(np.int32)
    w = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    got = oracle.moe("dequant", c.x, ids, w, c.wp, c.scale, g)
    ref = np.zeros((T, N))
    for t in range(T):
        for j in range(topk):
            e = ids[t, j]
            if 0 <= e < E:
                ref[t] += float(w[t, j]) * oracle.dequant(c.x[t:t + 1], c.wp[e], c.scale[e], g)[0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- bf16 activations (dequant form)

def _to_bf16_bits(v):
    """Round-to-nearest-even float32 -> bfloat16 bit patterns, done with
    numpy integer arithmetic on the float32 bits (independent of the oracle)."""
    b = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def test_bf16_decode_matches_float32_upper_half():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = oracle.bf16_to_double(bits)
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_dequant_bf16_matches_numpy_gemm():
    rng = np.random.default_rng(41)
    M, K, N, g = 5, 256, 40, 64
    c = make_case(M, K, N, g, seed=3)
    xb = _to_bf16_bits(rng.standard_normal((M, K)))
    sb = _to_bf16_bits(rng.uniform(-3, 3, (K // g, N)))
    x = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = (sb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = oracle.unpack_w(c.wp[0], K, N).astype(np.float64)
    ref = x @ (np.repeat(s, g, axis=0) * w)
    np.testing.assert_allclose(oracle.dequant_bf16(xb, c.wp[0], sb, g), ref, rtol=1e-12, atol=1e-9)


def test_dequant_bf16_equals_fp16_oracle_on_shared_values():
    """Values exact in both formats (small integers x, power-of-two scales)
    give the same y through the fp16 and the bf16 oracle."""
    rng = np.random.default_rng(43)
    M, K, N, g = 3, 128, 24, 32
    c = make_case(M, K, N, g, seed=4)
    xi = rng.integers(-8, 9, (M, K)).astype(np.float32)
    si = np.ldexp(1.0, rng.integers(-6, 2, (K // g, N))).astype(np.float32)
    y16 = oracle.dequant(xi.astype(np.float16), c.wp[0], si.astype(np.float16), g)
    yb = oracle.dequant_bf16(_to_bf16_bits(xi), c.wp[0], _to_bf16_bits(si), g)
    np.testing.assert_array_equal(y16, yb)


# ---------------------------------------------------------------- MSD with S unfold steps (reading R16)

def _golden_steps():
    with open(os.path.join(GOLDEN, "msd_worked_example_steps.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_worked_example_four_digits(mode):
    """The hand-worked example carried one residual step further: the fourth
    digit, its Y, and the 2- and 4-step outputs against their bounds."""
    ex, base = _golden_steps(), _golden()
    g = ex["g"]
    x = np.array([ex["x"]], dtype=np.float16)
    w = np.array(ex["w"], dtype=np.int8)
    scale = np.array([ex["scale"]], dtype=np.float16)
    amax, a = oracle.msd_expand_steps(x, g, 4, mode)
    assert amax[0, 0] == base["amax"]
    assert [a[i, 0].tolist() for i in range(4)] == [base["A1"], base["A2"], base["A3"], ex["A4"]]
    yint = oracle.msd_yint_planes(a, pack_int4(w), w.shape[1], g)
    assert [yint[i, 0, 0].tolist() for i in range(4)] == [base["Y1"], base["Y2"], base["Y3"], ex["Y4"]]
    for S, key in ((2, "2step"), (4, "4step")):
        y = oracle.msd_steps(x, pack_int4(w), scale, g, S, mode)
        np.testing.assert_allclose(y[0], ex["y_msd_" + key], rtol=1e-12, atol=0)
        assert np.all(np.abs(y[0] - np.array(base["y_exact"])) <= np.array(ex["truncation_bound_" + key]))


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_steps_are_prefixes_and_match_the_three_step_oracle(mode):
    """An S-step expansion's digits are the first S digits of a longer one
    (the recursion does not look ahead), and S = 3 equals the separately
    written three-step functions bit for bit (digits, A_max and y)."""
    rng = np.random.default_rng(21)
    for g in (32, 128):
        x = _adversarial_x(rng, 8, 512, g)
        amax4, a4 = oracle.msd_expand_steps(x, g, 4, mode)
        for S in (1, 2, 3):
            amax, a = oracle.msd_expand_steps(x, g, S, mode)
            assert np.array_equal(amax, amax4)
            assert np.array_equal(a, a4[:S])
        amax3, a3 = oracle.msd_expand(x, g, mode)
        assert np.array_equal(amax3, amax4) and np.array_equal(a3, a4[:3])
    c = make_case(5, 256, 40, 64, seed=5)
    assert np.array_equal(oracle.msd_steps(c.x, c.wp[0], c.scale[0], 64, 3, mode),
                          oracle.msd(c.x, c.wp[0], c.scale[0], 64, mode))


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
@pytest.mark.parametrize("S", [1, 2, 3, 4])
def test_steps_digits_and_reconstruction(mode, S):
    """Every digit |A_i| <= 7, and 7.49*x/A_max = sum_i A_i/14.98^(i-1) +
    r/14.98^(S-1) with |r| <= 0.5.  Binary32 adds the rounding of tmp1 (at
    most 7.49 * 2^-23 plus the gap between 7.49f and 7.49) once."""
    rng = np.random.default_rng(31 + S)
    g = 64
    x = _adversarial_x(rng, 8, 256, g)
    amax, a = oracle.msd_expand_steps(x, g, S, mode)
    assert np.abs(a).max() <= 7
    xd = x.astype(np.float64)
    am = np.repeat(amax, g, axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = np.where(am > 0, 7.49 * xd / am, 0.0)
    rec = sum(a[i] / 14.98 ** i for i in range(S))
    slack = 1e-12 if mode == oracle.MODE_FP64 else 2e-6
    assert np.abs(t - rec).max() <= 0.5 / 14.98 ** (S - 1) + slack


@pytest.mark.parametrize("mode", [oracle.MODE_FP32, oracle.MODE_FP64])
def test_steps_within_their_truncation_bounds_and_shrinking(mode):
    """y_S stays within sum_g A_max * 0.5/(7.49 * 14.98^(S-1)) * |scale| *
    sum|W| of the exact GEMM, and more steps give a smaller error (the
    accuracy side of the knob)."""
    g = 64
    c = make_case(6, 512, 80, g, seed=61, keep_w=True)
    c.x[2, :g] = 0
    ye = _exact_gemm(c.x, c.w[0], c.scale[0], g)
    K, N = c.w[0].shape
    absw = np.abs(c.w[0].astype(np.float64)).reshape(K // g, g, N).sum(axis=1)
    mag = None
    errs = []
    for S in (1, 2, 3, 4):
        amax, _ = oracle.msd_expand_steps(c.x, g, S, mode)
        mag = amax @ (np.abs(c.scale[0].astype(np.float64)) * absw)
        y = oracle.msd_steps(c.x, c.wp[0], c.scale[0], g, S, mode)
        bound = mag * 0.5 / (7.49 * 14.98 ** (S - 1))
        slack = 1e-12 if mode == oracle.MODE_FP64 else mag * 2e-6 / 7.49
        assert np.all(np.abs(y - ye) <= bound + slack)
        errs.append(np.abs(y - ye).max())
    assert errs[0] > errs[1] > errs[2] > errs[3] > 0


def test_yint_planes_match_integer_gemm_and_sampled_steps_match_full():
    c = make_case(4, 256, 48, 64, seed=78, keep_w=True)
    amax, a = oracle.msd_expand_steps(c.x, 64, 4)
    yint = oracle.msd_yint_planes(a, c.wp[0], 48, 64)
    w = c.w[0].astype(np.int64)
    for r in range(4):
        for gi in range(4):
            ref = a[r].astype(np.int64)[:, gi * 64:(gi + 1) * 64] @ w[gi * 64:(gi + 1) * 64]
            assert np.array_equal(yint[r, :, gi], ref)
    rows = np.array([0, 3, 1, 3, 2])
    cols = np.array([47, 0, 5, 9, 30])
    for S in (2, 4):
        full = oracle.msd_steps(c.x, c.wp[0], c.scale[0], 64, S)
        assert np.array_equal(oracle.msd_at_steps(c.x, c.wp[0], c.scale[0], 64, S, rows, cols), full[rows, cols])


def test_bf16_input_encoding_is_round_to_nearest_even():
    """The seeded bf16 inputs (inputs.to_bf16_bits) round float32 to the
    nearest bf16, ties to even, as torch's own float32 -> bfloat16 cast does,
    on random values and on every tie pattern of the low half-word."""
    import torch
    from inputs import to_bf16_bits
    rng = np.random.default_rng(17)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-38).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38], np.float32)])
    # ties: low half-word exactly 0x8000 above even and odd bf16 patterns
    hi = rng.integers(0x0080, 0x7F00, 500).astype(np.uint32)
    ties = ((hi << 16) | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(to_bf16_bits(v), ref)
