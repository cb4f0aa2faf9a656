"""The MSD expansion kernel rounds each digit step by adding and subtracting
1.5 * 2^23 in binary32 and takes the digit's byte from the sum's bits.  This
pins that identity on the host, in IEEE binary32 round-to-nearest-even (numpy
float32 arithmetic): for every |t| < 8 (a digit step never leaves that range)

    (t + 1.5*2^23) - 1.5*2^23 == rint(t)      (ties to even, exact)
    low byte of bits(t + 1.5*2^23) == int8(rint(t))

checked exhaustively around every half-integer in (-8, 8) and on a dense
random sample.  Section 4.1 of the MSD page (steps 3-7) defines the digits
with rint."""
import numpy as np
import pytest

MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def _check(t):
    t = np.asarray(t, dtype=np.float32)
    s = (t + MAGIC).astype(np.float32)
    a = (s - MAGIC).astype(np.float32)
    r = np.rint(t).astype(np.float32)
    assert np.array_equal(a, r), t[a != r][:8]
    low = (s.view(np.uint32) & 0xFF).astype(np.uint8)
    want = r.astype(np.int32).astype(np.int8).view(np.uint8)
    assert np.array_equal(low, want), t[low != want][:8]


def test_every_value_near_each_half_integer():
    # all binary32 values within 4096 ulps of k + 0.5 for k in [-8, 7], and
    # the integers themselves
    vals = []
    for k in range(-8, 8):
        c = np.float32(k + 0.5)
        bits = np.int64(np.float32(c).view(np.int32))
        span = np.arange(-4096, 4097, dtype=np.int64)
        vals.append((bits + span).astype(np.int32).view(np.float32))
        vals.append(np.float32(k))
    v = np.concatenate([np.atleast_1d(x) for x in vals])
    v = v[np.abs(v) < 8]
    _check(v)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_sample(seed):
    rng = np.random.default_rng(seed)
    t = rng.uniform(-8.0, 8.0, size=2_000_000).astype(np.float32)
    _check(t)
    # and small magnitudes, where the residual steps land
    _check((t * np.float32(1e-3)).astype(np.float32))


def test_signed_zero_gives_the_same_byte():
    _check(np.array([-0.0, 0.0, -0.25, 0.25, -0.5, 0.5], dtype=np.float32))
