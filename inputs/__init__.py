"""Seeded synthetic inputs for the A16W4 per-group matmul.

This module is shared by the tests and the benchmark: it only draws random
numbers and encodes them into the operator's input formats.  It holds none of
the method's arithmetic (no expansion, no matmul, no dequantisation), so both
the CPU oracle and the CUDA library can be fed from it without sharing code.

Input formats (the operator spec of "WeightQuantBatchMatmulExperiment 算子深度解析",
section 4.2 / 4.3):
  x      fp16 [M, K] row-major
  w      int4 [K, N], stored "two int4 per byte" as uint8 [K/2, N]: byte (i, n)
         holds W[2i, n] in the low nibble and W[2i+1, n] in the high nibble,
         two's complement
  scale  fp16 [K/g, N] (antiquant_scale, one per group of g rows of W and column)

Workloads (seed = 0x5EED0000 + index):
  0 msd_small   M=16   K=256  N=256   g=64   x[3, 64:128] forced to zero
  1 decode_m1   M=1    K=4096 N=4096  g=128
  2 decode_m16  M=16   K=4096 N=14336 g=128
  3 prefill     M=4096 K=4096 N=4096  g=128
  4 moe_e8      E=8 experts, T=4096 tokens, K=4096, N=14336, g=128
Value distributions: x ~ N(0,1) in fp16 with each entry multiplied by 20 with
probability 1e-3 (workload 4: no outliers); W uniform on the integers [-8, 7];
scale ~ U[0.005, 0.02] rounded to fp16.  Workload 4 draws per-expert token
counts from Multinomial(T, 1/E each) and sorts tokens by expert, described by
offsets[E+1] (exclusive prefix sums).

The page's own example (section 4.3: M=1, N=12288, K=8192, g=128, x ~ U[-3,3],
w in [-7,7], scale ~ U[-3,3]) is available as ``page_example``.

bf16 activations (the dequant variant's INT4 + BF16 pairing): ``make_case``
with ``act="bf16"`` draws the same distributions in float32 and encodes x and
scale as bfloat16 bit patterns (uint16, round to nearest even), the format's
definition being the upper 16 bits of a binary32.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

SEED_BASE = 0x5EED0000


@dataclass
class Workload:
    name: str
    M: int
    K: int
    N: int
    g: int
    E: int = 1
    outliers: bool = True
    zero_group: Optional[tuple] = None   # (row, k0, k1) forced to zero


WORKLOADS = [
    Workload("msd_small", 16, 256, 256, 64, zero_group=(3, 64, 128)),
    Workload("decode_m1", 1, 4096, 4096, 128),
    Workload("decode_m16", 16, 4096, 14336, 128),
    Workload("prefill", 4096, 4096, 4096, 128),
    Workload("moe_e8", 4096, 4096, 14336, 128, E=8, outliers=False),
]


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


def pack_int4(w: np.ndarray) -> np.ndarray:
    """int8 values in [-8, 7], shape [K, N] -> uint8 [K/2, N] (two per byte)."""
    w = np.asarray(w)
    assert w.shape[0] % 2 == 0
    u = w.astype(np.int8).view(np.uint8) & 0x0F
    return (u[0::2] | (u[1::2] << 4)).astype(np.uint8)


def to_bf16_bits(v) -> np.ndarray:
    """float32 values -> bfloat16 bit patterns (uint16), round to nearest even
    on the float32 bits (finite inputs)."""
    b = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _encode(v, act):
    return to_bf16_bits(np.asarray(v, np.float32)) if act == "bf16" else v.astype(np.float16)


def draw_x(rng, M, K, outliers=True, act="fp16") -> np.ndarray:
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outliers:
        mask = rng.random((M, K), dtype=np.float32) < 1e-3
        x = np.where(mask, x * 20.0, x)
    return _encode(x, act)


def draw_w(rng, K, N, lo=-8, hi=7) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=(K, N), dtype=np.int8)


def draw_scale(rng, G, N, lo=0.005, hi=0.02, act="fp16") -> np.ndarray:
    return _encode(rng.uniform(lo, hi, size=(G, N)), act)


@dataclass
class Case:
    x: np.ndarray                 # fp16 [M, K] (bf16 cases: uint16 bit patterns)
    wp: List[np.ndarray]          # per expert: uint8 [K/2, N]
    scale: List[np.ndarray]       # per expert: fp16 [K/g, N] (bf16 cases: uint16)
    g: int
    offsets: Optional[np.ndarray] = None   # int32 [E+1] (grouped only)
    w: List[np.ndarray] = field(default_factory=list)  # int8 [K, N] when kept

    @property
    def M(self):
        return self.x.shape[0]

    @property
    def K(self):
        return self.x.shape[1]

    @property
    def N(self):
        return self.wp[0].shape[1]

    @property
    def E(self):
        return len(self.wp)


def make_case(M, K, N, g, seed, E=1, outliers=True, zero_group=None,
              keep_w=False, grouped=None, act="fp16") -> Case:
    """Draw one problem.  ``grouped`` (default: E > 1) adds expert offsets;
    ``act`` = "fp16" or "bf16" (x and scale as bfloat16 bit patterns)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = draw_x(rng, M, K, outliers, act)
    if zero_group is not None:
        r, k0, k1 = zero_group
        x[r, k0:k1] = 0
    wps, scales, ws = [], [], []
    for _ in range(E):
        w = draw_w(rng, K, N)
        wps.append(pack_int4(w))
        scales.append(draw_scale(rng, K // g, N, act=act))
        if keep_w:
            ws.append(w)
    offsets = None
    if grouped if grouped is not None else E > 1:
        counts = rng.multinomial(M, np.full(E, 1.0 / E))
        offsets = np.zeros(E + 1, np.int32)
        offsets[1:] = np.cumsum(counts)
    return Case(x, wps, scales, g, offsets, ws)


def make_workload(name_or_index, keep_w=False, act="fp16") -> Case:
    idx = name_or_index if isinstance(name_or_index, int) else \
        [w.name for w in WORKLOADS].index(name_or_index)
    wl = WORKLOADS[idx]
    return make_case(wl.M, wl.K, wl.N, wl.g, SEED_BASE + idx, E=wl.E,
                     outliers=wl.outliers, zero_group=wl.zero_group, keep_w=keep_w, act=act)


def page_example(seed=SEED_BASE + 100, M=1, K=8192, N=12288, g=128) -> Case:
    """The page's own example distributions (section 4.3)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.uniform(-3, 3, size=(M, K)).astype(np.float16)
    w = draw_w(rng, K, N, -7, 7)
    scale = rng.uniform(-3, 3, size=(K // g, N)).astype(np.float16)
    return Case(x, [pack_int4(w)], [scale], g, None, [w])
