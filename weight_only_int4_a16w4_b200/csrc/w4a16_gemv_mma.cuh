// w4a16_gemv_mma.cuh -- the decode kernel for small batches on the warp-level
// tensor-core instructions (mma.sync), both variants.
//
// Operator: y = x . (antiquant_scale (.) W), "WeightQuantBatchMatmulExperiment
// 算子深度解析" (bjdmk.com.cn/news/4847346), section 4.1 (MSD, steps 9-11)
// and the plain dequant definition.  At a handful of tokens the matmul is a
// weight stream; what limits a CUDA-core dot product is the instruction count
// per weight, and the 5th-generation tcgen05 MMA, with only 16 tokens of N,
// costs far more to issue than the tile takes to compute.  The warp-level
// MMA takes its operands from registers, so each weight word goes from the
// load straight into an MMA fragment:
//
//  * B operand = the weights: one m16n8 MMA covers 8 output columns (an
//    "8-column block").  Lane (g, t) = (lane / 4, lane % 4) loads column g's
//    16-byte cell of piece 4q + t of a "quad" q (four 32-K pieces, 128 K;
//    the packed layout of repack_kernel: a cell is the 32 K values of one
//    column), and MMA j of the quad takes word j of every lane's cell, so one
//    quad of one block is four MMAs (MSD) or eight (dequant, K = 16 each).
//    The MMA sums over its K slots in any order, so mixing four pieces in one
//    MMA is exact as long as they share a group: groups are whole quads
//    (g % 128 == 0).
//  * MSD (m16n8k32, s8 x u8 -> s32): a word's bytes q & 0x0F0F0F0F and
//    (q >> 4) & 0x0F0F0F0F are the weights' u = w + 8 at K offsets
//    {0,4,1,5} / {2,6,3,7} of the word -- the fragment's two registers.  The
//    A rows are (digit plane i, token m), row i*M + m; lane (r, t)'s A
//    registers are words 2j, 2j+1 of plane i of piece 4q + t's digit record,
//    which gemv_expand_kernel writes in exactly this byte order.  Y_i = D -
//    8 * (sum of the quad's digits), exact in int32; per group the combine
//    (equations 9-11) Y_i * c_i * A_max * scale is added to an fp32 sum per
//    (row, column); the three planes of a token are added at the end.  With
//    S = 2 or 4 unfold steps the rows are the S planes of each token (S * M
//    <= 8) and the records carry S planes.
//  * DEQUANT (m16n8k16, f16 -> f32): a word unpacks to four fp16 pairs of the
//    exact weights (K offsets (0,1), (2,3), (4,5), (6,7)); the A rows are the
//    tokens and lane (m, t)'s A registers for word j are x[m][8j .. 8j+7] of
//    piece 4q + t, in natural order.  The fp32 sum of a group is multiplied
//    by its scale.
//  * DEQUANT with bf16 x, scale and y (m16n8k16, bf16 -> f32): the same, the
//    weights unpacked to exact bf16 pairs (int4_to_bf162x4).
//
// Work split: CTA c takes the 8-column blocks [c*B/P, (c+1)*B/P); warp w
// takes an even share of the quads of every block (a group may be cut: its
// running sum is closed at the group's end and at the warp's last quad); the
// warps' fp32 sums meet in shared memory and are added in warp order.  A
// round is one quad of four blocks (32 columns): for each of the quad's
// four pieces the warp copies the 32 columns' cells -- 512 contiguous bytes
// of the packed layout, lane l taking column l -- with cp.async into its
// ring in shared memory, at an XOR-swizzled slot so that the fragment reads
// (lane (g, t) takes the cell of column g of piece 4q + t) are free of bank
// conflicts.  Two rounds (dequant) or four (MSD) are in flight per warp, the
// first ones issued before the kernel waits for the previous grid
// (programmatic dependent launch), so the weight stream of a call overlaps
// the tail of the previous one.  The weights hold no registers in flight, so 16 warps of
// at most 64 registers keep enough loads outstanding (the memory system
// wants many warps with a few loads each).  A 32-warp instance (two rounds in
// flight per warp, one CTA per SM) serves wide dequant calls.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "sm100_ptx.cuh"
#include "w4a16_gemv.cuh"
#include "w4a16_kernels.cuh"

namespace w4a16 {

constexpr int kMgWarps = 16;                 // warps of the default instance (NW)
constexpr int kMgCB = 4;     // 8-column blocks per round (one cell per lane per piece)


template <int VAR, int MR, int NW = kMgWarps>
struct MgCfg {
    static constexpr int kWarps = NW;
    static constexpr int kThreads = NW * 32;
    static constexpr bool kIsMsd = is_msd(VAR);
    static constexpr bool kBf16 = VAR == kDeqBf16;
    static constexpr int kS = kIsMsd ? msd_steps(VAR) : 1;   // digit planes per token
    static constexpr int kRec = gemv_rec_words(kS);          // words per MSD record
    static constexpr int kRows = kS * MR;                    // A / D rows in use
    // rounds in flight per warp: 4 deep, the CTA alone on its SM (measured:
    // deeper rings beat keeping the next call's CTA resident, except for a
    // dequant call that only ever follows another dequant call)
    static constexpr int kDepth = NW >= 32 ? 2 : 4;
    static constexpr int kRing = kDepth * 4 * 512 + kDepth * kMgCB * 16;   // weight cells + scales, per warp
    static_assert(kRows <= 8, "rows must fit the lower half of the m16 tile");
    static constexpr int kRed = NW * kMgCB * kRows * 8 * 4;   // [warp][block][row][column] fp32
    static_assert(kMgCB * MR * 8 <= NW * 32, "the final sum needs a thread per (block, row, column)");
    // the most quads (and 32-K pieces) one warp takes
    __host__ __device__ static constexpr int qpw(int npieces) { return (npieces / 4 + NW - 1) / NW; }
    __host__ __device__ static constexpr int ppw(int npieces) { return 4 * qpw(npieces); }
    // one warp's operand: MSD the digit records of its pieces [ppw][M][kRec
    // words]; DEQUANT its slice of x [M][ppw * 32] fp16
    __host__ __device__ static constexpr int operand_bytes(int M, int npieces)
    {
        return kIsMsd ? ppw(npieces) * M * kRec * 4 : ppw(npieces) * M * 64;
    }
    __host__ __device__ static constexpr int warp_stride(int M, int npieces, int ppg)
    {
        return (void)ppg, kRing + operand_bytes(M, npieces);
    }
    __host__ __device__ static constexpr int smem_bytes(int M, int npieces, int ppg)
    {
        return kRed + NW * warp_stride(M, npieces, ppg);
    }
};

__device__ __forceinline__ uint32_t ldg_stream32(const void* p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// D += A . B on an m16n8k32 tile: A signed bytes, B unsigned bytes, int32
// sums.  The fragments are whole register tuples (a[1] and a[3], rows 8-15,
// stay zero), so no moves are needed around the instruction.
__device__ __forceinline__ void mma_s8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A . B on an m16n8k16 tile, fp16 in, fp32 sums
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A . B on an m16n8k16 tile, bf16 in, fp32 sums
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// a pair of scales (fp16, or bf16 bit patterns) as floats
template <bool BF>
__device__ __forceinline__ float2 scale_pair(const __half* p)
{
    if constexpr (BF) return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    else return __half22float2(*reinterpret_cast<const __half2*>(p));
}

// Eight packed weights -> four fp16 pairs of the exact signed values, K
// offsets (0,1), (2,3), (4,5), (6,7): 0x6400 | u is 1024 + u and 0x6400 |
// (u << 4) is 1024 + 16u in binary16 (u = w + 8), so w = (1024 + u) - 1032 =
// (1024 + 16u) / 16 - 72, each exact.
__device__ __forceinline__ void unpack_exact_f16(uint32_t q, uint32_t (&p)[4])
{
    const uint32_t q8 = q >> 8;
    const __half2 b1032 = __half2half2(__ushort_as_half(0x6408u));   // 1032
    const __half2 s16 = __half2half2(__ushort_as_half(0x2C00u));     // 1/16
    const __half2 b72 = __half2half2(__ushort_as_half(0xD480u));     // -72
    const uint32_t r0 = (q & 0x000F000Fu) | 0x64006400u;
    const uint32_t r1 = (q & 0x00F000F0u) | 0x64006400u;
    const uint32_t r2 = (q8 & 0x000F000Fu) | 0x64006400u;
    const uint32_t r3 = (q8 & 0x00F000F0u) | 0x64006400u;
    const __half2 w0 = __hsub2(*reinterpret_cast<const __half2*>(&r0), b1032);
    const __half2 w1 = __hfma2(*reinterpret_cast<const __half2*>(&r1), s16, b72);
    const __half2 w2 = __hsub2(*reinterpret_cast<const __half2*>(&r2), b1032);
    const __half2 w3 = __hfma2(*reinterpret_cast<const __half2*>(&r3), s16, b72);
    p[0] = *reinterpret_cast<const uint32_t*>(&w0);
    p[1] = *reinterpret_cast<const uint32_t*>(&w1);
    p[2] = *reinterpret_cast<const uint32_t*>(&w2);
    p[3] = *reinterpret_cast<const uint32_t*>(&w3);
}

template <int VAR, int MR, int NW, bool DBG = false>
__global__ void __launch_bounds__(NW * 32, NW >= 32 ? 1 : 2) gemv_mma_kernel(const __grid_constant__ GemvParams P)
{
    using C = MgCfg<VAR, MR, NW>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gl = lane >> 2, tl = lane & 3;   // fragment row / column group of this lane
    const int M = P.M, K = P.K;
    const int ppg = P.g / 32, qpg = ppg / 4;   // pieces and quads per group
    const int ppw = C::ppw(P.npieces);
    float* red = reinterpret_cast<float*>(smem);   // [warp][block][row][column]
    uint8_t* wreg = smem + C::kRed + warp * C::warp_stride(M, P.npieces, ppg);
    uint8_t* ring = wreg;                                               // [depth][piece][32 cells], swizzled
    uint8_t* sring = wreg + C::kDepth * 4 * 512;                         // [depth][block] 8 fp16 scales
    const uint8_t* opnd = wreg + C::kRing;
    const uint32_t* rec_w = reinterpret_cast<const uint32_t*>(opnd);    // MSD: [ppw][M][kRec]
    const __half* xw = reinterpret_cast<const __half*>(opnd);           // DEQUANT: [M][ppw * 32]

    // (the host keeps nblk * ctas below 2^31)
    const int b0 = static_cast<int>((blockIdx.x * static_cast<unsigned>(P.nblk)) / static_cast<unsigned>(P.ctas));
    const int b1 = static_cast<int>(((blockIdx.x + 1) * static_cast<unsigned>(P.nblk)) / static_cast<unsigned>(P.ctas));
    const int nq = P.npieces / 4;
    const int qw0 = (warp * nq) / NW, qw1 = ((warp + 1) * nq) / NW;
    const int pw0 = 4 * qw0, pw1 = 4 * qw1;
    const int rpb = C::qpw(P.npieces);                  // rounds per block-group (same for every warp)
    const int gw0 = qw0 / qpg, qpos0 = qw0 - gw0 * qpg;  // the warp's first group, its quads before qw0
    const int nbg = (b1 - b0 + kMgCB - 1) / kMgCB;
    const int nitems = nbg * rpb;

    // this lane's A row: MSD (plane, token) = (gl / M, gl % M); DEQUANT token
    // gl.  A lane past the real rows reads a valid row anyway: its MMA rows
    // are never read back.
    const bool row_ok = gl < C::kS * M;
    int row_m, row_plane;
    if constexpr (C::kIsMsd) {
        // the instance's MR fixes M: MR = 1 -> M = 1, MR = 2 -> M = 2,
        // MR = 4 -> M = 3 or 4
        if constexpr (MR == 1) {
            row_m = 0;
            row_plane = gl;
        } else if constexpr (MR == 2) {
            row_m = M == 1 ? 0 : (gl & 1);
            row_plane = M == 1 ? gl : (gl >> 1);
        } else {
            row_m = M == 4 ? (gl & 3) : gl % 3;
            row_plane = M == 4 ? (gl >> 2) : gl / 3;
        }
        row_plane = min(row_plane, C::kS - 1);
    } else {
        row_m = gl < M ? gl : 0;
        row_plane = 0;
    }
    // combine weight 1 / (7.49 * 14.98^plane) of this lane's row
    const float row_c = (C::kS <= 3 || row_plane < 3) ? (row_plane == 0 ? kC1 : (row_plane == 1 ? kC2 : kC3)) : kC4;

    // the next kernel in the stream may start its own weight stream now
    griddep_launch_dependents();

    // round (bg, rr) -> ring slot `slot`: quad q = qw0 + rr of the 32
    // columns of block-group bg; lane l copies column l's cell of each of the
    // quad's pieces j to cell slot l ^ 2j of piece row j, lanes 0..3 the 8
    // scales of block `lane` for the quad's group.  One commit group per
    // round, empty or not.
    auto load = [&](int slot, int bg, int rr, int grp) {
        const int q = qw0 + rr;
        const int c = (b0 + bg * kMgCB) * 8 + lane;   // this lane's column
        if (bg < nbg && q < qw1) {
            if (c < b1 * 8) {
                const uint8_t* src = P.w + (static_cast<size_t>(c >> 7) * P.kchunks + q) * kWStage + (c & 127) * 16;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    cp_async16(smem_addr(ring + (slot * 4 + j) * 512 + ((lane ^ (2 * j)) * 16)), src + j * 2048);
            }
            const int b = b0 + bg * kMgCB + lane;
            if (lane < kMgCB && b < b1 && !DBG)
                cp_async16(smem_addr(sring + (slot * kMgCB + lane) * 16),
                           P.scale + static_cast<size_t>(grp) * P.N + b * 8);
        }
        cp_async_commit();
    };

    using Acc = typename std::conditional<C::kIsMsd, int, float>::type;
    Acc d[kMgCB][4];        // the open group's running MMA sums (rows 8-15 unused)
    float acc[kMgCB][2];    // closed groups, scaled
    uint32_t af[4] = {0u, 0u, 0u, 0u};   // A fragments; [1] and [3] (rows 8-15) stay zero
    uint32_t ag[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < kMgCB; ++k) {
        d[k][0] = d[k][1] = d[k][2] = d[k][3] = Acc(0);
        acc[k][0] = acc[k][1] = 0.f;
    }
    int corr = 0;           // MSD: -8 * (digit sum) of the open group's quads, this lane's row
    int gpos = 0;           // quads of the open group done

    auto compute = [&](int slot, int bg, int rr) {
        const int bb = b0 + bg * kMgCB;
        const int nbk = min(kMgCB, b1 - bb);
        if (rr == 0) gpos = qpos0;
        const int q = qw0 + rr;
        if (q < qw1) {
            const bool closes = ++gpos == qpg || q + 1 == qw1;
            if (gpos == qpg) gpos = 0;
            // word j of this lane's cell of block k (column 8k + gl, piece 4q + tl)
            const uint32_t* cellw = reinterpret_cast<const uint32_t*>(ring + (slot * 4 + tl) * 512);
            auto cword = [&](int k, int j) { return cellw[((8 * k + gl) ^ (2 * tl)) * 4 + j]; };
            const __half* sg = reinterpret_cast<const __half*>(sring + slot * kMgCB * 16) + 2 * tl;
            if constexpr (C::kIsMsd) {
                // lane (row, tl) reads the record of piece 4q + tl
                const uint32_t* r = rec_w + ((4 * rr + tl) * M + row_m) * C::kRec;
                int c = static_cast<int>(r[8 * C::kS + row_plane]);
                if (!row_ok) c = 0;
                c += __shfl_xor_sync(0xffffffffu, c, 1);
                c += __shfl_xor_sync(0xffffffffu, c, 2);
                corr += c;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    af[0] = r[row_plane * 8 + 2 * j];
                    af[2] = r[row_plane * 8 + 2 * j + 1];
#pragma unroll
                    for (int k = 0; k < kMgCB; ++k) {
                        if (k >= nbk) break;
                        const uint32_t w = cword(k, j);
                        mma_s8u8(d[k], af, w & 0x0F0F0F0Fu, (w >> 4) & 0x0F0F0F0Fu);
                    }
                }
                if (closes) {
                    if constexpr (DBG) {
                        // the warp's part of the group's Y_i (a group may be cut
                        // between two warps: the window adds the parts exactly)
                        if (row_ok) {
                            const int grp = (4 * q) / ppg;
#pragma unroll
                            for (int k = 0; k < kMgCB; ++k) {
                                if (k >= nbk) break;
                                const int n = (bb + k) * 8 + 2 * tl;
                                dbg_put_yint<true>(P, row_plane, row_m, grp, n, d[k][0] + corr);
                                dbg_put_yint<true>(P, row_plane, row_m, grp, n + 1, d[k][1] + corr);
                            }
                            const int nb0 = P.dbg_n0 / 8;
                            if (row_plane == 0 && tl == 0 && nb0 >= bb && nb0 < bb + nbk && row_m >= P.dbg_m0 &&
                                row_m < P.dbg_m1)
                                P.dbg_amax[static_cast<size_t>(row_m - P.dbg_m0) * P.G + grp] =
                                    __uint_as_float(r[9 * C::kS]);
                        }
                    }
                    // word 9S of a record is the A_max of its group
                    const float alpha = row_ok ? row_c * __uint_as_float(r[9 * C::kS]) : 0.f;   // rows past S M: unused
#pragma unroll
                    for (int k = 0; k < kMgCB; ++k) {
                        if (k >= nbk) break;
                        const float2 s = __half22float2(*reinterpret_cast<const __half2*>(sg + k * 8));
                        // exact int32 -> fp32 (|Y| < 2^22)
                        const float y0 = __int2float_rn(d[k][0] + corr);
                        const float y1 = __int2float_rn(d[k][1] + corr);
                        acc[k][0] = fmaf(y0, alpha * s.x, acc[k][0]);
                        acc[k][1] = fmaf(y1, alpha * s.y, acc[k][1]);
                        d[k][0] = d[k][1] = d[k][2] = d[k][3] = 0;
                    }
                    corr = 0;
                }
            } else {
                const uint32_t* xr = reinterpret_cast<const uint32_t*>(xw + row_m * ppw * 32 + (4 * rr + tl) * 32);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // x[8j .. 8j+3] and x[8j+4 .. 8j+7] of this lane's piece
                    af[0] = xr[4 * j];
                    af[2] = xr[4 * j + 1];
                    ag[0] = xr[4 * j + 2];
                    ag[2] = xr[4 * j + 3];
#pragma unroll
                    for (int k = 0; k < kMgCB; ++k) {
                        if (k >= nbk) break;
                        uint32_t wp[4];
                        if constexpr (C::kBf16) {
                            int4_to_bf162x4(cword(k, j), wp);
                            mma_bf16(d[k], af, wp[0], wp[1]);
                            mma_bf16(d[k], ag, wp[2], wp[3]);
                        } else {
                            unpack_exact_f16(cword(k, j), wp);
                            mma_f16(d[k], af, wp[0], wp[1]);
                            mma_f16(d[k], ag, wp[2], wp[3]);
                        }
                    }
                }
                if (closes) {
#pragma unroll
                    for (int k = 0; k < kMgCB; ++k) {
                        if (k >= nbk) break;
                        const float2 s = scale_pair<C::kBf16>(sg + k * 8);
                        acc[k][0] = fmaf(d[k][0], s.x, acc[k][0]);
                        acc[k][1] = fmaf(d[k][1], s.y, acc[k][1]);
                        d[k][0] = d[k][1] = d[k][2] = d[k][3] = 0.f;
                    }
                }
            }
        }
        // after the block-group's last round: add the warps' sums in warp
        // order (and, for MSD, the three digit planes of each token), write y
        if (rr == rpb - 1) {
            if (gl < C::kRows) {
#pragma unroll
                for (int k = 0; k < kMgCB; ++k) {
                    float* r = red + ((warp * kMgCB + k) * C::kRows + gl) * 8 + 2 * tl;
                    r[0] = acc[k][0];
                    r[1] = acc[k][1];
                }
            }
            __syncthreads();
            // thread (k, m, col) = (tid / (8 MR), (tid / 8) % MR, tid % 8)
            const int k = tid / (8 * MR), m = (tid >> 3) % MR, col = tid & 7;
            if (k < nbk && m < M) {
                const float* r = red + (k * C::kRows) * 8 + col;
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const float* rw = r + w * kMgCB * C::kRows * 8;
                    if constexpr (C::kIsMsd) {
                        float t = rw[m * 8];
#pragma unroll
                        for (int p = 1; p < C::kS; ++p) t += rw[(p * M + m) * 8];
                        s += t;
                    } else {
                        s += rw[m * 8];
                    }
                }
                if (!DBG) store_elem<C::kBf16>(P.y + static_cast<size_t>(m) * P.N + (bb + k) * 8 + col, s);
            }
            if (bg + 1 < nbg) __syncthreads();
#pragma unroll
            for (int k2 = 0; k2 < kMgCB; ++k2) acc[k2][0] = acc[k2][1] = 0.f;
        }
    };

    // rounds 0 .. depth-1 before the wait; the load cursor carries the
    // round's block-group, quad index and the quad's group (position in it)
    int lbg = 0, lrr = 0, lgrp = gw0, lgpos = qpos0;
    auto advance_load = [&]() {
        if (++lgpos == qpg) {
            lgpos = 0;
            ++lgrp;
        }
        if (++lrr == rpb) {
            lrr = 0;
            ++lbg;
            lgrp = gw0;
            lgpos = qpos0;
        }
    };
#pragma unroll
    for (int s = 0; s < C::kDepth; ++s) {
        load(s, lbg, lrr, lgrp);
        advance_load();
    }

    // x and the MSD records (and whatever wrote them) are valid once the
    // previous grid is done; each warp copies only its own pieces' operand
    griddep_wait();
    const int npw = pw1 - pw0;
    if constexpr (C::kIsMsd) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(P.rec + static_cast<size_t>(pw0) * M * C::kRec);
        const int nv = npw * M * (C::kRec / 4);
        for (int v = lane; v < nv; v += 32) cp_async16(smem_addr(opnd + v * 16), src + v * 16);
    } else {
        // row m's slice: npw * 4 vectors of 16 bytes
        for (int m = 0; m < M; ++m)
            for (int e = lane; e < npw * 4; e += 32)
                cp_async16(smem_addr(opnd + (m * ppw * 4 + e) * 16), P.x + static_cast<size_t>(m) * K + pw0 * 32 + e * 8);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncwarp();

    int cbg = 0, crr = 0;   // next round to compute
    for (int i = 0; i < nitems; ++i) {
        const int slot = i % C::kDepth;
        compute(slot, cbg, crr);
        if (++crr == rpb) {
            crr = 0;
            ++cbg;
        }
        // the slot is free again: refill it, then wait for the next round
        __syncwarp();
        load(slot, lbg, lrr, lgrp);
        advance_load();
        cp_async_wait<C::kDepth - 1>();
        __syncwarp();
    }
}

}  // namespace w4a16
