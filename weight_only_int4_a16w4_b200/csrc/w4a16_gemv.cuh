// w4a16_gemv.cuh -- the decode kernel for the smallest batches (M <= 4):
// a GEMV on the CUDA cores, both variants.
//
// Operator: y = x . (antiquant_scale (.) W), "WeightQuantBatchMatmulExperiment
// 算子深度解析" (bjdmk.com.cn/news/4847346), section 4.1 (MSD, steps 1-11)
// and the plain dequant definition.  At M <= 4 the matmul is a stream of
// weights with a handful of multiply-adds per weight: a 128 x 16 tensor-core
// tile would be mostly padding, so the CUDA cores do the arithmetic and the
// kernel is shaped around getting every weight byte in flight at once.
//
// Work split: output columns only.  The columns form blocks of 32 (one warp
// width); CTA c of P takes blocks [c*B/P, (c+1)*B/P) and all of K, so no
// partial sums leave the CTA.  Inside a CTA warp w takes a contiguous run of
// whole groups (G/8 of them) of the block, lane l owns column 32*b + l, and
// a shared-memory sum over the 8 warps (in warp order) gives y.  Sums stay
// per group (integer Y_i for MSD) until the group's last piece, where the
// scale (and A_max) is applied once.  Every lane
// loads its weights as 16-byte vectors straight into registers (a warp reads
// 512 contiguous bytes of the packed layout, see repack_kernel): two rounds
// of eight loads per thread are issued before the kernel waits for the
// previous grid, so the weight stream of this call overlaps the tail of the
// previous one (programmatic dependent launch).
//
// MSD: gemv_expand_kernel runs first and writes, once per call, A_max and
// the digits A1..A3 (section 4.1 steps 1-8, the same IEEE binary32 steps as
// expand_kernel) as one record per (32-K piece, row): the digit bytes in the
// order the packed weight words unpack to, so that each weight word meets
// its digits in two dp4a per digit plane: Y_i = sum_k (w+8) * A_i -
// 8 * sum_k A_i, exact in int32.  Per piece, (Y1/7.49 + Y2/(7.49*14.98) +
// Y3/(7.49*14.98^2)) * A_max * scale is added to the column's fp32 sum
// (equations 9-11: a group's pieces add up to its Y_i, and the combine is
// linear in Y_i).
//
// DEQUANT: each weight word gives four fp16 pairs of biased values (1024 + u
// or 1024 + 16u, exact) that meet x through the mixed-precision
// fma.rn.f32.f16 (exact products, fp32 sums); one correction per piece made
// from the sums of x removes the biases, and the group scale multiplies
// each piece's sum.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"
#include "w4a16_kernels.cuh"

namespace w4a16 {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvRound = 8;                        // 16-byte loads per thread per round
constexpr int kGemvRecWords = 28;                    // MSD record: 24 digit words, 3 sums, A_max
// record of an MSD call with S digit planes: 8 S digit words, S sums, A_max,
// padded to whole 16-byte vectors (S = 3: 28 words)
__host__ __device__ constexpr int gemv_rec_words(int S) { return (9 * S + 1 + 3) / 4 * 4; }
constexpr int kGemvMaxMK = 32768;                    // M * K bound of the shared-memory operand

struct GemvParams {
    const __half* x;          // [M][K]
    const uint8_t* w;         // packed blocks
    const __half* scale;      // [G][N]
    __half* y;                // [M][N]
    const uint32_t* rec;      // MSD: [K/32][M][28] digit records
    int M, K, N, g, G;
    int kchunks;              // ceil(K / 128)
    int npieces;              // K / 32
    int nblk;                 // ceil(N / 32)
    int ctas;                 // P
    // MSD Y_int debug window (DBG instances only): int32 [S][m1-m0][G][n1-n0]
    // and A_max fp32 [m1-m0][G]; no scale is read and no y is written
    int32_t* dbg_yint;
    float* dbg_amax;
    int dbg_m0, dbg_m1, dbg_n0, dbg_n1;
};

// One MSD Y_i (plane p of token m, group grp, column n) into the debug
// window, if it lies there.  ATOMIC: a group's sum arrives in parts (from
// several warps) and is added up exactly in int32 (the window starts at 0).
template <bool ATOMIC>
__device__ __forceinline__ void dbg_put_yint(const GemvParams& P, int p, int m, int grp, int n, int y)
{
    if (m < P.dbg_m0 || m >= P.dbg_m1 || n < P.dbg_n0 || n >= P.dbg_n1) return;
    const int wm = P.dbg_m1 - P.dbg_m0, wn = P.dbg_n1 - P.dbg_n0;
    int32_t* dst = P.dbg_yint + ((static_cast<size_t>(p) * wm + (m - P.dbg_m0)) * P.G + grp) * wn + (n - P.dbg_n0);
    if (ATOMIC) atomicAdd(dst, y);
    else *dst = y;
}

template <int VAR, int MR>
struct GemvCfg {
    static constexpr bool kIsMsd = VAR == kMsd;
    static constexpr int kRed = kGemvWarps * MR * 32 * 4;   // cross-warp sum buffer
    __host__ __device__ static constexpr int operand_bytes(int M, int K)
    {
        // MSD: the digit records; DEQUANT: x as fp16 and one fp32
        // bias correction per (32-K piece, row)
        return kIsMsd ? (K / 32) * M * kGemvRecWords * 4 : M * K * 2 + (K / 32) * M * 4;
    }
    __host__ __device__ static constexpr int smem_bytes(int M, int K)
    {
        return kRed + ((operand_bytes(M, K) + 15) / 16) * 16;
    }
};

// unsigned bytes of `a` times signed bytes of `b`, summed into c
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// c + a.lo * b.lo + a.hi * b.hi, fp16 inputs, products exact, fp32 adds
__device__ __forceinline__ float fma2_f16_f32(uint32_t a2, uint32_t b2, float c)
{
    float d;
    asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t.reg .f32 t;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 t, al, bl, %3;\n\t"
        "fma.rn.f32.f16 %0, ah, bh, t;\n\t}"
        : "=f"(d)
        : "r"(a2), "r"(b2), "f"(c));
    return d;
}

// Eight packed weights -> four fp16 pairs holding biased values, exactly:
// from the binary16 format, 0x6400 | u is 1024 + u and 0x6400 | (u << 4) is
// 1024 + 16u (u = w + 8), so p0 = 1024 + (u0, u1), p1 = 1024 + 16 (u2, u3),
// p2 = 1024 + (u4, u5), p3 = 1024 + 16 (u6, u7).  The biases are removed once
// per piece (see gemv_kernel), not per weight.
__device__ __forceinline__ void gemv_unpack_biased(uint32_t q, uint32_t (&p)[4])
{
    const uint32_t q8 = q >> 8;
    p[0] = (q & 0x000F000Fu) | 0x64006400u;
    p[1] = (q & 0x00F000F0u) | 0x64006400u;
    p[2] = (q8 & 0x000F000Fu) | 0x64006400u;
    p[3] = (q8 & 0x00F000F0u) | 0x64006400u;
}

// 16 bytes of the weight stream, read once: not kept in L1
__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ------------------------------------------------------------------ MSD steps 1-8 for the GEMV

// One warp per (row m, span of max(g, 128) K values); lane l holds the
// values 4l .. 4l+3 of each 128-value sub-chunk of the span (NSUB = span /
// 128 sub-chunks).  A_max per group (g < 128: the g/4 lanes of a group reduce
// among themselves), then the S digits in IEEE binary32 with the literal
// operation order of steps 2-7, then per 32-K piece (8 lanes) a record of
// R = gemv_rec_words(S) words (28 for S = 3): word i*8 + 2j + h holds digit
// plane i's bytes for the piece's packed word j, low (h = 0: K offsets 8j +
// {0, 4, 1, 5}) or high (h = 1: 8j + {2, 6, 3, 7}) nibbles -- the byte order
// of q & 0x0F0F0F0F and (q >> 4) & 0x0F0F0F0F for a packed word q; words
// 8S .. 9S-1 hold -8 * (sum of the piece's digits of plane i) and word 9S the
// A_max of the piece's group (fp32 bits).  rec: [K/32][M][R].
// Digits and record of one 128-K sub-chunk of one row (steps 2-8 in IEEE
// binary32, the literal operation order): lane l holds the sub-chunk's values
// 4l .. 4l+3 in v and am, the A_max of their group; every lane takes part in
// the shuffles, and lanes with `store` write the record of their 32-K piece
// (lane / 8) at r.
template <int S>
__device__ __forceinline__ void msd_subchunk_record(const float (&v)[4], float am, int lane, uint32_t* r, bool store)
{
    uint32_t word[S];
    int sum[S];
#pragma unroll
    for (int i = 0; i < S; ++i) {
        word[i] = 0u;
        sum[i] = 0;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (am != 0.f) {
            float t = __fdiv_rn(__fmul_rn(7.49f, v[e]), am);
#pragma unroll
            for (int i = 0; i < S; ++i) {
                const float a = rintf(t);
                const int d = static_cast<int>(a);
                word[i] |= (static_cast<uint32_t>(d) & 0xFFu) << (8 * e);
                sum[i] += d;
                if (i + 1 < S) t = __fmul_rn(__fsub_rn(t, a), 14.98f);
            }
        }
    }
    // lanes 2j and 2j+1 of each 8-lane piece hold K offsets 8j..8j+3 and 8j+4..8j+7
#pragma unroll
    for (int i = 0; i < S; ++i) {
        const uint32_t other = __shfl_xor_sync(0xffffffffu, word[i], 1);
        // even lane: [a0 a4 a1 a5] from (mine = a0..a3, other = a4..a7);
        // odd lane:  [a2 a6 a3 a7] from (other = a0..a3, mine = a4..a7)
        const uint32_t out = (lane & 1) ? __byte_perm(other, word[i], 0x7362) : __byte_perm(word[i], other, 0x5140);
        int t = sum[i];
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        t += __shfl_xor_sync(0xffffffffu, t, 4);
        if (store) {
            r[i * 8 + (lane & 7)] = out;
            if ((lane & 7) == 0) r[8 * S + i] = static_cast<uint32_t>(-8 * t);
        }
    }
    // a piece lies inside one group (g % 32 == 0)
    if (store && (lane & 7) == 0) r[9 * S] = __float_as_uint(am);
}

template <int NSUB, int S>
__global__ void __launch_bounds__(256) gemv_expand_kernel(const __half* __restrict__ x, int M, int K, int g,
                                                          uint32_t* __restrict__ rec)
{
    constexpr int R = gemv_rec_words(S);
    // the matmul that reads the records may launch now and stream its
    // weights; x may come from the previous kernel, and the previous matmul
    // may still read the records this kernel overwrites
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int span = NSUB * kKC;
    const int nspans = (K + span - 1) / span;
    const long long wg = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
    if (wg >= static_cast<long long>(M) * nspans) return;
    const int m = static_cast<int>(wg / nspans), sp = static_cast<int>(wg % nspans);

    float v[NSUB][4];
    float am = 0.f;
#pragma unroll
    for (int s = 0; s < NSUB; ++s) {
        const int k0 = sp * span + s * kKC + 4 * lane;
        if (k0 < K) {
            const uint2 raw = *reinterpret_cast<const uint2*>(x + static_cast<size_t>(m) * K + k0);
            const __half2 x01 = *reinterpret_cast<const __half2*>(&raw.x);
            const __half2 x23 = *reinterpret_cast<const __half2*>(&raw.y);
            v[s][0] = __low2float(x01);
            v[s][1] = __high2float(x01);
            v[s][2] = __low2float(x23);
            v[s][3] = __high2float(x23);
        } else {
            v[s][0] = v[s][1] = v[s][2] = v[s][3] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(v[s][e]));
    }
    // A_max of each group: g >= 128 spans the warp's whole span; g < 128
    // covers g/4 consecutive lanes; every lane ends with its group's value
    const int lanes_per_group = g >= kKC ? 32 : g / 4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
        if (o < lanes_per_group) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));

#pragma unroll
    for (int s = 0; s < NSUB; ++s) {
        const int k0 = sp * span + s * kKC + 4 * lane;
        const int pg = (sp * span + s * kKC) / 32 + (lane >> 3);
        // a piece lies wholly inside or outside K (K % 32 == 0)
        msd_subchunk_record<S>(v[s], am, lane, rec + (static_cast<size_t>(pg) * M + m) * R, k0 < K);
    }
}

// ------------------------------------------------------------------ the GEMV

template <int VAR, int MR, bool DBG = false>
__global__ void __launch_bounds__(kGemvThreads, 2) gemv_kernel(const __grid_constant__ GemvParams P)
{
    using C = GemvCfg<VAR, MR>;
    extern __shared__ __align__(16) uint8_t smem[];
    float* red = reinterpret_cast<float*>(smem);                        // [8 warps][MR][32]
    uint8_t* operand = smem + C::kRed;
    const int rec_words = P.npieces * P.M * kGemvRecWords;
    const uint32_t* rec_s = reinterpret_cast<const uint32_t*>(operand);
    const __half* xs = reinterpret_cast<const __half*>(operand);
    float* xcorr = reinterpret_cast<float*>(operand + P.M * P.K * 2);   // DEQUANT: [K/32][M]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int M = P.M, K = P.K;
    const int b0 = static_cast<int>((static_cast<long long>(blockIdx.x) * P.nblk) / P.ctas);
    const int b1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * P.nblk) / P.ctas);
    // warp w takes the whole groups [w*G/8, (w+1)*G/8), i.e. a contiguous run
    // of 32-K pieces [pw0, pw1); a group is ppg pieces
    const int ppg = P.g / 32;
    const int pw0 = ((warp * P.G) / kGemvWarps) * ppg;
    const int pw1 = (((warp + 1) * P.G) / kGemvWarps) * ppg;
    // rounds per column block: the same for every warp (the block-end sum
    // below is a CTA-wide barrier), sized for the warp with the most groups
    const int rpb = (((P.G + kGemvWarps - 1) / kGemvWarps) * ppg + kGemvRound - 1) / kGemvRound;
    const int nitems = (b1 - b0) * rpb;

    // the next kernel in the stream may start its own weight stream now
    griddep_launch_dependents();

    // round i: column block b0 + i / rpb, pieces pw0 + 8 * (i % rpb) + j; the
    // scale of a group is loaded with its last piece (two per register: piece
    // j's in the low / high half of sc[j / 2])
    auto load = [&](uint4 (&buf)[kGemvRound], uint32_t (&sc)[kGemvRound / 2], int i) {
        const int b = b0 + i / rpb, rr = i % rpb;
        const int n = b * 32 + lane;
        const int tile = n >> 7, r = n & 127;
        const uint8_t* wt = P.w + static_cast<size_t>(tile) * P.kchunks * kWStage + r * 16;
        const int pbase = pw0 + kGemvRound * rr;
        int grp = pbase / ppg, pos = (kGemvRound * rr) % ppg;   // group of the next piece, pieces done in it
#pragma unroll
        for (int j = 0; j < kGemvRound; ++j) {
            const int p = pbase + j;
            uint32_t h = 0u;
            if (p < pw1) {
                buf[j] = ldg_stream(wt + static_cast<size_t>(p >> 2) * kWStage + (p & 3) * 2048);
                if (++pos == ppg) {
                    if (n < P.N && !DBG) h = __half_as_ushort(P.scale[static_cast<size_t>(grp) * P.N + n]);
                    ++grp;
                    pos = 0;
                }
            }
            if (j & 1)
                sc[j >> 1] |= h << 16;
            else
                sc[j >> 1] = h;
        }
    };

    float acc[MR];
    int yacc[MR][3];       // MSD: the group's Y1..Y3 so far
    float gsum[MR];        // DEQUANT: the group's sum_k x w so far
#pragma unroll
    for (int m = 0; m < MR; ++m) {
        acc[m] = 0.f;
        gsum[m] = 0.f;
        yacc[m][0] = yacc[m][1] = yacc[m][2] = 0;
    }

    auto compute = [&](const uint4 (&buf)[kGemvRound], const uint32_t (&sc)[kGemvRound / 2], int i) {
        const int rr = i % rpb;
        const int pbase = pw0 + kGemvRound * rr;
        int grp = pbase / ppg, pos = (kGemvRound * rr) % ppg;
#pragma unroll
        for (int j = 0; j < kGemvRound; ++j) {
            const int p = pbase + j;
            if (p >= pw1) break;
            const uint32_t q[4] = {buf[j].x, buf[j].y, buf[j].z, buf[j].w};
            const bool group_end = ++pos == ppg;
            if constexpr (C::kIsMsd) {
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    lo[t] = q[t] & 0x0F0F0F0Fu;
                    hi[t] = (q[t] >> 4) & 0x0F0F0F0Fu;
                }
#pragma unroll
                for (int m = 0; m < MR; ++m) {
                    if (m >= M) break;
                    const uint4* r4 =
                        reinterpret_cast<const uint4*>(rec_s + (static_cast<size_t>(p) * M + m) * kGemvRecWords);
                    const uint4 ini = r4[6];
                    const int init[3] = {static_cast<int>(ini.x), static_cast<int>(ini.y), static_cast<int>(ini.z)};
#pragma unroll
                    for (int pl = 0; pl < 3; ++pl) {
                        const uint4 d0 = r4[pl * 2], d1 = r4[pl * 2 + 1];
                        int a = yacc[m][pl] + init[pl];
                        a = dp4a_us(lo[0], d0.x, a);
                        a = dp4a_us(hi[0], d0.y, a);
                        a = dp4a_us(lo[1], d0.z, a);
                        a = dp4a_us(hi[1], d0.w, a);
                        a = dp4a_us(lo[2], d1.x, a);
                        a = dp4a_us(hi[2], d1.y, a);
                        a = dp4a_us(lo[3], d1.z, a);
                        a = dp4a_us(hi[3], d1.w, a);
                        yacc[m][pl] = a;
                    }
                }
                if (group_end) {
                    const float scl =
                        __half2float(__ushort_as_half(static_cast<unsigned short>(sc[j >> 1] >> (16 * (j & 1)))));
                    if constexpr (DBG) {
                        // warps take whole groups: yacc is the group's Y_i
                        const int n = (b0 + i / rpb) * 32 + lane;
#pragma unroll
                        for (int m = 0; m < MR; ++m) {
                            if (m >= M) break;
#pragma unroll
                            for (int pl = 0; pl < 3; ++pl) dbg_put_yint<false>(P, pl, m, grp, n, yacc[m][pl]);
                            if (n == P.dbg_n0 && m >= P.dbg_m0 && m < P.dbg_m1)
                                P.dbg_amax[static_cast<size_t>(m - P.dbg_m0) * P.G + grp] =
                                    __uint_as_float(rec_s[(static_cast<size_t>(p) * M + m) * kGemvRecWords + 27]);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < MR; ++m) {
                        if (m >= M) break;
                        const float v = fmaf(static_cast<float>(yacc[m][2]), kC3,
                                             fmaf(static_cast<float>(yacc[m][1]), kC2,
                                                  static_cast<float>(yacc[m][0]) * kC1));
                        // word 27 of a record is the A_max of its group
                        const float amx = __uint_as_float(rec_s[(static_cast<size_t>(p) * M + m) * kGemvRecWords + 27]);
                        acc[m] = fmaf(v, amx * scl, acc[m]);
                        yacc[m][0] = yacc[m][1] = yacc[m][2] = 0;
                    }
                    ++grp;
                    pos = 0;
                }
            } else {
                // with A = K offsets {0,1,4,5} and B = {2,3,6,7} of each word,
                // s1 = sum_A x (1024 + u) and s16 = sum_B x (1024 + 16u), so the
                // piece's sum_k x w = s1 + s16 / 16 - 1032 X_A - 72 X_B, the
                // last two terms (sums of x alone) precomputed per piece
                uint32_t h[4][4];
#pragma unroll
                for (int t = 0; t < 4; ++t) gemv_unpack_biased(q[t], h[t]);
#pragma unroll
                for (int m = 0; m < MR; ++m) {
                    if (m >= M) break;
                    const uint4* x4 = reinterpret_cast<const uint4*>(xs + static_cast<size_t>(m) * K + p * 32);
                    float s1a = 0.f, s1b = 0.f, s16a = 0.f, s16b = 0.f;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint4 xv = x4[t];             // x[8t .. 8t+7] as four pairs
                        s1a = fma2_f16_f32(xv.x, h[t][0], s1a);
                        s16a = fma2_f16_f32(xv.y, h[t][1], s16a);
                        s1b = fma2_f16_f32(xv.z, h[t][2], s1b);
                        s16b = fma2_f16_f32(xv.w, h[t][3], s16b);
                    }
                    gsum[m] += (s1a + s1b) + fmaf(s16a + s16b, 0.0625f, xcorr[p * M + m]);
                }
                if (group_end) {
                    const float scl =
                        __half2float(__ushort_as_half(static_cast<unsigned short>(sc[j >> 1] >> (16 * (j & 1)))));
#pragma unroll
                    for (int m = 0; m < MR; ++m) {
                        acc[m] = fmaf(gsum[m], scl, acc[m]);
                        gsum[m] = 0.f;
                    }
                    pos = 0;
                }
            }
        }
        // after the block's last round: sum the 8 warps in order, write y
        if (rr == rpb - 1) {
#pragma unroll
            for (int m = 0; m < MR; ++m) red[(warp * MR + m) * 32 + lane] = acc[m];
            __syncthreads();
            if (tid < 32 * MR) {
                const int m = tid >> 5, l = tid & 31;
                const int n = (b0 + i / rpb) * 32 + l;
                if (m < M && n < P.N && !DBG) {
                    float s = 0.f;
#pragma unroll
                    for (int w = 0; w < kGemvWarps; ++w) s += red[(w * MR + m) * 32 + l];
                    P.y[static_cast<size_t>(m) * P.N + n] = __float2half_rn(s);
                }
            }
            __syncthreads();
#pragma unroll
            for (int m = 0; m < MR; ++m) acc[m] = 0.f;
        }
    };

    uint4 bufA[kGemvRound], bufB[kGemvRound];
    uint32_t scA[kGemvRound / 2], scB[kGemvRound / 2];
    if (nitems > 0) load(bufA, scA, 0);
    if (nitems > 1) load(bufB, scB, 1);

    // x and the MSD records (and whatever wrote them) are valid once the
    // previous grid is done
    griddep_wait();
    if constexpr (C::kIsMsd) {
        const uint4* src = reinterpret_cast<const uint4*>(P.rec);
        uint4* dst = reinterpret_cast<uint4*>(operand);
        for (int v = tid; v < rec_words / 4; v += kGemvThreads) dst[v] = src[v];
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(P.x);
        uint4* dst = reinterpret_cast<uint4*>(operand);
        for (int v = tid; v < M * K / 8; v += kGemvThreads) dst[v] = src[v];
        __syncthreads();
        // per (piece, row): -(1032 X_A + 72 X_B), X_A / X_B the sums of x over
        // the offsets {0,1,4,5} / {2,3,6,7} of each 8-value word
        for (int v = tid; v < P.npieces * M; v += kGemvThreads) {
            const int pc = v / M, m = v % M;
            const uint4* x4 = reinterpret_cast<const uint4*>(xs + static_cast<size_t>(m) * K + pc * 32);
            float xa = 0.f, xb = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint4 xv = x4[t];
                const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&xv.x));
                const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&xv.y));
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&xv.z));
                const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&xv.w));
                xa += (f0.x + f0.y) + (f2.x + f2.y);
                xb += (f1.x + f1.y) + (f3.x + f3.y);
            }
            xcorr[v] = -fmaf(1032.f, xa, 72.f * xb);
        }
    }
    __syncthreads();

    for (int i = 0; i < nitems; i += 2) {
        compute(bufA, scA, i);
        if (i + 2 < nitems) load(bufA, scA, i + 2);
        if (i + 1 < nitems) {
            compute(bufB, scB, i + 1);
            if (i + 3 < nitems) load(bufB, scB, i + 3);
        }
    }
}

}  // namespace w4a16
