// w4a16_kernels.cuh -- the device side of the A16W4 per-group matmul.
//
// Operator: y = x . (antiquant_scale (.) W), "WeightQuantBatchMatmulExperiment
// 算子深度解析" (bjdmk.com.cn/news/4847346), sections 4.1-4.3.
//
// Kernels
//   repack_kernel   offline int4 re-layout (the "Marlin layout" idea,
//                   pwwt.cn/news/2290475 section 6.2; QUICK's offline
//                   interleave, briefgpt.xyz "QUICK" abstract).
//   expand8_kernel / expand_kernel   MSD equations 1-8: A_max and the residual digits A1..A3
//                   (section 4.1, steps 1-8), written once to HBM.
//   gemm_kernel     the tensor-core matmul, both variants, dense / split-K /
//                   grouped-expert.  MSD: equations 9-11; DEQUANT: y = x.W'.
//
// gemm_kernel is "swap-AB": the weight tile is the 128-row MMA operand A
// (rows = 128 output columns n, held in Tensor Memory), the activations are
// operand B (rows = tokens, K-major in shared memory, brought by TMA), and
// the accumulator D is [128 n][tokens] in Tensor Memory.  For MSD the three
// residual matrices are stacked along the MMA N dimension (3 x TT rows of B),
// the B200 analogue of stacking A1..A3 into a 3M-row A_int (section 4.1
// step 8; section 8.1 "singleCoreM = 3*M"), so one MMA produces Y1, Y2, Y3.
//
// Warp roles (the counts are template parameters; GemmCfg below):
//   warp 0      weight producer: bulk copies of the packed weight chunks
//               (and the fp16 scale rows when the converter applies them)
//               into a ring of shared-memory slots; four chunks per copy on
//               the decode tile.
//   warp 1      activation producer (TMA tiles of x, or of the digit planes,
//               into the operand stages) and Tensor Memory allocation.
//   warps 2..   MMA issuers: one lane each issues the tcgen05 MMAs of its
//               chunks and commits them to the stage / accumulator barriers.
//   converters  groups of 4 warps: shared-memory int4 -> MMA operand A in
//               Tensor Memory (int8 for MSD, fp16 or bf16 for DEQUANT), one
//               thread per weight row, written with tcgen05.st.
//   epilogue    groups of 4 warps: tcgen05.ld of the accumulators; MSD
//               combines Y1..Y3 with A_max and the scale after every group
//               (equations 10-11) while the MMAs of the next group run (the
//               PRELOAD_MSD overlap of section 6.2, done with multi-buffered
//               accumulators); fp16 / bf16 store or split-K partial.
#pragma once

#ifndef W4A16_ROLE_UNROLL
#define W4A16_ROLE_UNROLL _Pragma("unroll")
#endif

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace w4a16 {

constexpr int kBN = 128;                 // output columns per tile (MMA M)
constexpr int kKC = 128;                 // K per pipeline stage
constexpr int kWStage = kBN * kKC / 2;   // packed bytes per (tile, chunk): 8192
constexpr int kMaxExperts = 64;
constexpr int kMaxGroupMsd = 512;        // expand_kernel: at most 16 values per lane
// Decode tile: chunks per bulk copy of weights, and per tensor copy of
// activations when the map allows it.  Fewer, larger copies: the producers
// otherwise issue one chunk's copies per loop pass, and a pass costs far more
// than its few instructions (about 0.4 us per chunk measured on B200).
constexpr int kWCopyGroup = 4;          // weight chunks per bulk copy
constexpr int kBCopyGroup = 4;          // activation chunks per tensor copy

// kDeqBf16: the dequant variant with bf16 x, scale and y (the INT4 + BF16
// pairing of the Humming article, aihirek.info).  Its buffers travel in the
// same __half-typed fields as bit patterns; the kernels read them as bf16.
// kMsd2 / kMsd4: MSD with 2 or 4 unfold steps instead of 3 (the residual
// recursion of section 4.1 run for S digits; section 7 of the same page notes
// that the gain varies with the number of MSD unfold steps).
enum Variant { kMsd = 0, kDeq = 1, kDeqBf16 = 2, kMsd2 = 3, kMsd4 = 4 };

__host__ __device__ constexpr bool is_msd(int v) { return v == kMsd || v == kMsd2 || v == kMsd4; }
// digits per activation: 3 for the page's algorithm, 2 or 4 for the others
__host__ __device__ constexpr int msd_steps(int v) { return v == kMsd2 ? 2 : (v == kMsd4 ? 4 : 3); }

// Combine weights of equation 10 (denominators read as 7.49, 7.49*14.98,
// 7.49*14.98^2: the page prints them with the multiplication sign lost).
constexpr float kC1 = static_cast<float>(1.0 / 7.49);
constexpr float kC2 = static_cast<float>(1.0 / (7.49 * 14.98));
constexpr float kC3 = static_cast<float>(1.0 / (7.49 * 14.98 * 14.98));
constexpr float kC4 = static_cast<float>(1.0 / (7.49 * 14.98 * 14.98 * 14.98));
// combine weight of digit plane p (0-based): 1 / (7.49 * 14.98^p)
__host__ __device__ constexpr float msd_plane_c(int p) { return p == 0 ? kC1 : p == 1 ? kC2 : p == 2 ? kC3 : kC4; }

struct GemmParams {
    int M;          // dense: rows of x; grouped: total tokens T
    int K, N, g, G;
    int kchunks;    // ceil(K / 128)
    int n_tiles;    // ceil(N / 128)
    int t_slots;    // grid.z: token tiles (dense) or tile slots (grouped)
    int splits;     // split-K factor (dense); 1 = no split
    int unit;       // chunks per split unit (keeps splits on group boundaries)
    int issuers;    // MMA issuer warps in use (1 or 2)
    int E;
    const int32_t* offsets;                 // grouped: device [E+1]; dense: nullptr
    const uint8_t* w[kMaxExperts];          // packed weights per expert
    const __half* scale[kMaxExperts];       // [G][N] per expert
    __half* y;                              // [M][N]
    // routed form with one expert per token: row r of the grouped result goes
    // to y row row_dst[r], times the gate weight row_w[row_dst[r]]; nullptr:
    // row r to row r
    const int32_t* row_dst;
    const float* row_w;
    const float* amax;                      // MSD: [G][M]
    uint32_t* status;
    unsigned long long timeout_ns;
    int write_y;
    // decode tile: chunks per activation copy (1, or kBCopyGroup when the
    // tensor map spans kBCopyGroup chunks per box: dense calls, K % 128 == 0)
    int bgroup;
    int32_t* dbg_yint;                      // MSD debug window (or nullptr)
    float* dbg_amax;
    int dbg_m0, dbg_m1, dbg_n0, dbg_n1;
};

// Compile-time shape of one gemm_kernel instance.
//   TT     tokens per tile (MMA N for DEQUANT, N / 3 for MSD)
//   ST     operand stages: the converted A operand of a chunk in Tensor
//          Memory (and, except on the decode tile, its activation tile in
//          shared memory; the decode tile keeps 16 activation stages)
//   WST    weight stages (shared memory only): the packed weight chunk and
//          (optionally) its scale rows; deeper than ST so that enough weight
//          bytes are in flight while Tensor Memory bounds ST
//   NCONV  converter warp groups (4 warps each) taking alternate chunks
//   NEPI   epilogue warp groups (4 warps each) splitting the tile's tokens
//   NISS   MMA issuer warps available (the launch may use fewer)
//   SEPI   DEQUANT only: apply the group scale in the epilogue, to per-group
//          fp32 accumulators (decode tiles), instead of in the converter
//          (W' = fp16(scale * w), one accumulator over all of K)
//   DBG    write the MSD Y_int debug window
// Warps: 0 weight producer; 1 activation producer; 2 .. 1+NISS MMA issuers;
// the control block is padded to a multiple of 4 warps; then the converter
// groups, then the epilogue groups.  Chunk i lives in stage i % ST and is
// served by converter group i % NCONV and issuer i % issuers; ST is a
// multiple of both, so every stage is always served by the same group and no
// waiter can run two phases ahead of a barrier.  Group-accumulator mode keeps
// NBUF = max(2, NISS) accumulator buffers, buffer = group % NBUF; with several
// issuers a group is one chunk, so each issuer owns one buffer.
template <int VAR, int TT, int ST, int WST, int NCONV, int NEPI, int NISS, bool SEPI>
struct GemmCfg {
    static constexpr bool kIsMsd = is_msd(VAR);
    static constexpr bool kBf16 = VAR == kDeqBf16;
    static constexpr bool kGroupAcc = kIsMsd || SEPI;      // per-group accumulators + per-group epilogue
    static constexpr int kVals = kIsMsd ? msd_steps(VAR) : 1;   // accumulators per token (Y1..YS or y)
    static constexpr int kMmaN = kVals * TT;
    static constexpr int kBBytes = kIsMsd ? kVals * TT * 128 : 2 * TT * 128;   // activation tile per stage
    static constexpr int kSBytes = (kIsMsd || SEPI) ? 0 : 1024;            // up to 4 scale rows
    static constexpr int kStage = kBBytes;                                 // activation stage (shared memory)
    // activation stages: on the decode tile the tiles are small and every
    // CTA reads the same ones from L2, so a deep ring of their own keeps the
    // L2 latency off the MMA's path; elsewhere one per operand stage
    static constexpr int kBST = TT == 16 ? 16 : ST;
    static constexpr int kWSlot = kWStage + kSBytes;                       // weight stage
    // weight chunks per bulk copy: a tile's packed blocks of consecutive
    // chunks are contiguous, so with no scale rows in the slots one copy
    // fills several (decode tile)
    static constexpr int kWG = (TT == 16 && kSBytes == 0 && WST % kWCopyGroup == 0) ? kWCopyGroup : 1;
    static constexpr int kMaxIssuers = NISS;
    // accumulator buffers: per group (two, or one per issuer); a single
    // accumulator over all of K otherwise, one per issuer (added up, in
    // issuer order, by the epilogue)
    static constexpr int kNBuf = kGroupAcc ? (NISS > 2 ? NISS : 2) : NISS;
    static constexpr int kAccStride = ((kMmaN + 31) / 32) * 32;
    static constexpr int kAccCols = kNBuf * kAccStride;
    static constexpr int kACols = kIsMsd ? 32 : 64;                        // A operand per stage
    static constexpr int kColsUsed = kAccCols + ST * kACols;
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
    static constexpr int kCtrlWarps = ((2 + NISS + 3) / 4) * 4;
    static constexpr int kConvWarp0 = kCtrlWarps;
    static constexpr int kEpiWarp0 = kCtrlWarps + 4 * NCONV;
    static constexpr int kWarps = kCtrlWarps + 4 * NCONV + 4 * NEPI;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kEpiThreads = 128 * NEPI;
    // decode tile with several epilogue groups: group eg takes the K groups
    // j = eg, eg + NEPI, ... for all TT tokens (the per-group work is short
    // and latency-bound, so groups in flight overlap); otherwise the groups
    // split the tokens
    static constexpr bool kEpiRR = TT == 16 && NEPI > 1;
    static constexpr int kTokPerEpi = kEpiRR ? TT : TT / NEPI;
    // MSD epilogue with at most 48 sums per thread and group: read them all,
    // hand the buffer back, then combine
    static constexpr bool kEpiBurst = kIsMsd && kTokPerEpi * kVals <= 48;
    static constexpr int kRedBytes = TT == 16 ? TT * kBN * 4 + 256 : 0;     // split-K partials (decode tile only)
    static constexpr int kRRBytes = kEpiRR ? (NEPI - 1) * TT * kBN * 4 : 0; // partial sums of groups 1..NEPI-1
    static constexpr int kNumBars = 2 * kBST + 2 * ST + 2 * WST + 2 * kNBuf + kMaxIssuers;
    static constexpr int kSmem = kBST * kStage + WST * kWSlot + kRedBytes + kRRBytes + 1024 + 8 * kNumBars + 16 +
                                 4 * NEPI * 2 * TT * 4 + 16;
    static_assert(kColsUsed <= 512, "Tensor Memory overflow");
    static_assert(kMmaN % 16 == 0 && kMmaN >= 16 && kMmaN <= 256, "MMA N out of range");
    static_assert(TT % 16 == 0 && kTokPerEpi % 16 == 0, "token tile must split into 16-token pieces");
    static_assert(kStage % 1024 == 0 && kWSlot % 1024 == 0, "stages must keep 1024-byte alignment");
    static_assert(kSmem <= 227 * 1024, "shared memory overflow");
    static_assert(ST % NCONV == 0 && ST % NISS == 0 && WST % NCONV == 0 && kBST % NISS == 0,
                  "stages must split evenly over the groups");
    static_assert(TT != 16 || kBST % kBCopyGroup == 0, "grouped activation copies never wrap the ring");
    static_assert(NISS == 1 || NISS == 2 || NISS == 4, "1, 2 or 4 MMA issuers");
    static_assert(!SEPI || !kIsMsd, "SEPI is a DEQUANT option");
    // bf16 keeps 8 significant bits: a product scale * w does not fit, so the
    // weights stay exact and the scale is applied to the fp32 group sums
    static_assert(!kBf16 || SEPI, "the bf16 variant applies the scale in the epilogue");
    static_assert(!kEpiRR || (kGroupAcc && kNBuf % NEPI == 0), "round-robin epilogue needs per-group buffers");
};

// two fp32 lanes at once (sm_100 packed fp32): a * b + c and a * b, each lane
// rounded as the scalar instruction would
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t pack_half2_bits(__half2 h)
{
    return *reinterpret_cast<uint32_t*>(&h);
}

// Eight int4 weights of one packed word -> four fp16 pairs (w exactly).
// Word layout (written by repack_kernel): bits 4i..4i+3 (i < 4) hold element
// 2i, bits 16+4i.. hold element 2i+1, each as u = w + 8.  From the binary16
// format: 0x6400 | u is the half 1024 + u, and 0x6400 | (u << 4) is
// 1024 + 16u.  So pair 0 is (0x6400|u) - 1032 and pair 1 is
// (0x6400|16u) * (1/16) - 72, both exact (one rounding of an exact value);
// pairs 2 and 3 repeat this on the word shifted by 8.  9 instructions.
__device__ __forceinline__ void int4_to_half2x4(uint32_t q, uint32_t* out4)
{
    const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));   // 1032
    const __half2 k16th = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));   // 1/16
    const __half2 km72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));    // -72
    const uint32_t q8 = q >> 8;
    uint32_t h0 = (q & 0x000F000Fu) | 0x64006400u;
    uint32_t h1 = (q & 0x00F000F0u) | 0x64006400u;
    uint32_t h2 = (q8 & 0x000F000Fu) | 0x64006400u;
    uint32_t h3 = (q8 & 0x00F000F0u) | 0x64006400u;
    const __half2 w0 = __hsub2(*reinterpret_cast<__half2*>(&h0), k1032);
    const __half2 w1 = __hfma2(*reinterpret_cast<__half2*>(&h1), k16th, km72);
    const __half2 w2 = __hsub2(*reinterpret_cast<__half2*>(&h2), k1032);
    const __half2 w3 = __hfma2(*reinterpret_cast<__half2*>(&h3), k16th, km72);
    out4[0] = pack_half2_bits(w0);
    out4[1] = pack_half2_bits(w1);
    out4[2] = pack_half2_bits(w2);
    out4[3] = pack_half2_bits(w3);
}

// The same, each pair multiplied by the group scale: fp16(scale * w).
__device__ __forceinline__ void int4_to_half2x4_scaled(uint32_t q, __half2 s2, uint32_t* out4)
{
    int4_to_half2x4(q, out4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 v = __hmul2(*reinterpret_cast<__half2*>(&out4[i]), s2);
        out4[i] = pack_half2_bits(v);
    }
}

// Eight int4 weights of one packed word -> four bf16 pairs (w exactly), the
// same K offsets as int4_to_half2x4.  bfloat16 is the upper half of a
// binary32 (8 exponent bits, 7 fraction bits), so 0x4300 | u is 128 + u
// (the fraction's unit at 128 is 1) and (128 + u) - 136 = w is exact.  A
// nibble above bit 3 of a half would reach the exponent, so each pair is
// shifted down first.  11 instructions.
__device__ __forceinline__ void int4_to_bf162x4(uint32_t q, uint32_t* out4)
{
    const __nv_bfloat162 k136 = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h = ((q >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
        const __nv_bfloat162 w = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&h), k136);
        out4[i] = *reinterpret_cast<const uint32_t*>(&w);
    }
}

// One scale element of a call: fp16, or (BF) the bf16 bit pattern kept in
// the same 16 bits.
template <bool BF>
__device__ __forceinline__ float load_elem(const __half* p)
{
    if constexpr (BF) return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p)) << 16);
    else return __half2float(*p);
}

// One y element, rounded to nearest even: fp16, or (BF) bf16.
template <bool BF>
__device__ __forceinline__ void store_elem(__half* p, float v)
{
    if constexpr (BF) *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
    else *p = __float2half_rn(v);
}

// Row r of a tile's result, column n: stored at its own row, or (routed form,
// one expert per token) at its token's row times the token's gate weight.

template <bool BF>
__device__ __forceinline__ void store_row(const GemmParams& P, int r, int n, float v)
{
    if (P.row_dst == nullptr) {
        store_elem<BF>(P.y + static_cast<size_t>(r) * P.N + n, v);
        return;
    }
    const int dst = __ldg(P.row_dst + r);
    if (dst >= 0) store_elem<BF>(P.y + static_cast<size_t>(dst) * P.N + n, v * __ldg(P.row_w + dst));
}

// Eight int4 weights of one packed word -> two words of four signed int8 in
// K order (elements 0..3, then 4..7).
__device__ __forceinline__ void int8_word(uint32_t q, uint32_t* out2)
{
    const uint32_t lo = q & 0x0F0F0F0Fu;          // elements 0, 4, 1, 5
    const uint32_t hi = (q >> 4) & 0x0F0F0F0Fu;   // elements 2, 6, 3, 7
    const uint32_t a = __byte_perm(lo, hi, 0x6420);
    const uint32_t b = __byte_perm(lo, hi, 0x7531);
    // per byte: (u + 0x78) ^ 0x80 == u - 8 (mod 256); no carry crosses bytes
    out2[0] = (a + 0x78787878u) ^ 0x80808080u;
    out2[1] = (b + 0x78787878u) ^ 0x80808080u;
}

// ------------------------------------------------------------------ repack

// Logical bytes [K/2][N] -> kernel layout.  Block (n_tile, kc) of 8192 bytes
// holds rows n_tile*128 + r, K range kc*128 .. +127, as four 2048-byte
// pieces p (K sub-range 32p .. 32p+31); row r's 16 bytes of piece p sit at
// p*2048 + r*16 so that 128 threads read a piece conflict-free; word j of
// those 16 bytes holds K offsets 8j .. 8j+7 in the nibble order described
// at dequant_word, stored as w + 8.  Padding rows / columns hold w = 0.
__global__ void repack_kernel(const uint8_t* __restrict__ wl, int K, int N, int kchunks, int n_tiles,
                              uint32_t* __restrict__ out)
{
    const long long total = static_cast<long long>(n_tiles) * kchunks * 2048;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(idx & 3);
        const int r = static_cast<int>((idx >> 2) & 127);
        const int p = static_cast<int>((idx >> 9) & 3);
        const long long blk = idx >> 11;
        const int kc = static_cast<int>(blk % kchunks);
        const int nt = static_cast<int>(blk / kchunks);
        const int n = nt * kBN + r;
        const int kbase = kc * kKC + 32 * p + 8 * j;
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int k = kbase + e;
            uint32_t u = 8;   // w = 0
            if (n < N && k < K) {
                const uint8_t b = wl[static_cast<size_t>(k >> 1) * N + n];
                u = ((k & 1) ? (b >> 4) : b) & 0xF;
                u ^= 8u;      // two's complement nibble -> w + 8
            }
            const int pos = (e & 1) ? 4 + (e >> 1) : (e >> 1);
            word |= u << (4 * pos);
        }
        out[idx] = word;
    }
}

// ------------------------------------------------------------------ MSD expansion (eq. 1-8)

// One warp per (row m, group gi); lane l owns VPL = g/32 consecutive values.
// Arithmetic in IEEE binary32 with correctly rounded * / - and round to
// nearest even, in the order of equations 2-7:
//   tmp1 = (7.49f * x) / A_max; A1 = rint(tmp1)
//   tmp2 = (tmp1 - A1) * 14.98f; A2 = rint(tmp2)
//   tmp3 = (tmp2 - A2) * 14.98f; A3 = rint(tmp3)
// and, with S != 3 unfold steps, the same recursion for S digits.
// A_max == 0 gives zero digits.  Output: xq [S][M][K] int8 (equation 8's
// A_int, residual-major), amax [G][M] fp32.
template <int VPL, int S>
__global__ void __launch_bounds__(256) expand_kernel(const __half* __restrict__ x, int M, int K, int g,
                                                     int8_t* __restrict__ xq, float* __restrict__ amax)
{
    const int G = K / g;
    // Let the matmul that consumes A_int launch now (it streams its weights
    // meanwhile); x may come from the previous kernel, and the previous
    // matmul may still read the A_int this kernel overwrites, so wait for it.
    griddep_launch_dependents();
    griddep_wait();
    const long long warp = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= static_cast<long long>(M) * G) return;
    const int m = static_cast<int>(warp / G);
    const int gi = static_cast<int>(warp % G);
    const size_t base = static_cast<size_t>(m) * K + static_cast<size_t>(gi) * g + lane * VPL;

    float v[VPL];
    if constexpr (VPL % 4 == 0) {
        // 8-byte loads (VPL consecutive halves, 8-byte aligned: K % 32 == 0)
#pragma unroll
        for (int i = 0; i < VPL; i += 4) {
            const uint2 raw = *reinterpret_cast<const uint2*>(x + base + i);
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            v[i] = lo.x;
            v[i + 1] = lo.y;
            v[i + 2] = hi.x;
            v[i + 3] = hi.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) v[i] = __half2float(x[base + i]);
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) am = fmaxf(am, fabsf(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));

    int8_t d[S][VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        if (am == 0.f) {
#pragma unroll
            for (int p = 0; p < S; ++p) d[p][i] = 0;
        } else {
            float t = __fdiv_rn(__fmul_rn(7.49f, v[i]), am);
#pragma unroll
            for (int p = 0; p < S; ++p) {
                const float a = rintf(t);
                d[p][i] = static_cast<int8_t>(a);
                if (p + 1 < S) t = __fmul_rn(__fsub_rn(t, a), 14.98f);
            }
        }
    }
    const size_t plane = static_cast<size_t>(M) * K;
    if constexpr (VPL % 4 == 0) {
        // one 4-byte store per plane and 4 digits (4-byte aligned)
#pragma unroll
        for (int i = 0; i < VPL; i += 4) {
#pragma unroll
            for (int p = 0; p < S; ++p) {
                uint32_t wd = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) wd |= (static_cast<uint32_t>(static_cast<uint8_t>(d[p][i + e]))) << (8 * e);
                *reinterpret_cast<uint32_t*>(xq + p * plane + base + i) = wd;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i)
#pragma unroll
            for (int p = 0; p < S; ++p) xq[p * plane + base + i] = d[p][i];
    }
    if (lane == 0) amax[static_cast<size_t>(gi) * M + m] = am;
}

// The same steps for g <= 256, shaped for memory-level parallelism.  A thread
// takes 8 consecutive values (one 16-byte load) of the activations read as
// one flat [M * K] array, so LPG = g / 8 threads share a group (A_max by a
// shuffle over them; K % g == 0 keeps every group inside one row).  A warp
// task is STEPS consecutive 256-value blocks whose loads are all issued
// before any arithmetic; warps loop over tasks.  Each digit is rounded by
// adding and subtracting 1.5 * 2^23: for |t| < 2^22 the sum falls where
// binary32 values are the integers, so round-to-nearest-even there is rint(t)
// and the subtraction is exact (every step here has |t| < 8).  The digit's
// byte is then the low byte of the sum's bits (0x4B400000 + d).
__device__ __forceinline__ uint32_t low_bytes4(float a, float b, float c, float d)
{
    const uint32_t lo = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040);
    const uint32_t hi = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

template <int LPG, int S, int STEPS>
__global__ void __launch_bounds__(256) expand8_kernel(const __half* __restrict__ x, int M, int K, int g,
                                                      int8_t* __restrict__ xq, float* __restrict__ amax)
{
    static_assert(LPG == 4 || LPG == 8 || LPG == 16 || LPG == 32, "g = 8 * LPG, 32 <= g <= 256");
    // as expand_kernel: the consumer may launch now; wait for the producer of
    // x and for the previous reader of xq
    griddep_launch_dependents();
    griddep_wait();
    const int G = K / g;
    const long long total8 = static_cast<long long>(M) * K / 8;    // 8-value vectors
    const long long ntask = (total8 + 32 * STEPS - 1) / (32 * STEPS);
    const int lane = threadIdx.x & 31;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const size_t plane = static_cast<size_t>(M) * K;
    constexpr float kMagic = 12582912.0f;                          // 1.5 * 2^23
    for (long long task = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; task < ntask;
         task += nwarps) {
        uint4 raw[STEPS];
#pragma unroll
        for (int st = 0; st < STEPS; ++st) {
            const long long v = (task * STEPS + st) * 32 + lane;
            raw[st] = v < total8 ? __ldg(reinterpret_cast<const uint4*>(x + v * 8)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int st = 0; st < STEPS; ++st) {
            const long long v = (task * STEPS + st) * 32 + lane;
            float f[8];
            {
                const uint32_t w[4] = {raw[st].x, raw[st].y, raw[st].z, raw[st].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
                    f[2 * h] = t.x;
                    f[2 * h + 1] = t.y;
                }
            }
            float am = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(f[i]));
#pragma unroll
            for (int o = LPG / 2; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (v >= total8) continue;       // whole groups lie past the end
            float sv[S][8];                  // 1.5 * 2^23 + digit
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float t = am == 0.f ? 0.f : __fdiv_rn(__fmul_rn(7.49f, f[i]), am);
#pragma unroll
                for (int p = 0; p < S; ++p) {
                    sv[p][i] = __fadd_rn(t, kMagic);
                    if (p + 1 < S) t = __fmul_rn(__fsub_rn(t, __fsub_rn(sv[p][i], kMagic)), 14.98f);
                }
            }
#pragma unroll
            for (int p = 0; p < S; ++p)
                *reinterpret_cast<uint2*>(xq + p * plane + v * 8) =
                    make_uint2(low_bytes4(sv[p][0], sv[p][1], sv[p][2], sv[p][3]),
                               low_bytes4(sv[p][4], sv[p][5], sv[p][6], sv[p][7]));
            if (lane % LPG == 0) {
                const long long f0 = (v * 8) / g;                     // flat group index = m * G + gi
                amax[static_cast<size_t>(f0 % G) * M + f0 / G] = am;
            }
        }
    }
}

// ------------------------------------------------------------------ the tensor-core matmul

struct TileCoord {
    int n_tile, split, e, t0, t_end;
};

__device__ __forceinline__ bool resolve_tile(const GemmParams& P, int TT, TileCoord& c)
{
    c.n_tile = blockIdx.x;
    c.split = blockIdx.y;
    if (P.offsets == nullptr) {
        c.e = 0;
        c.t0 = blockIdx.z * TT;
        c.t_end = min(P.M, c.t0 + TT);
        return c.t_end > c.t0;
    }
    int slot = blockIdx.z;
    for (int e = 0; e < P.E; ++e) {
        const int a = min(max(__ldg(P.offsets + e), 0), P.M);
        const int b = min(max(__ldg(P.offsets + e + 1), a), P.M);
        const int nt = (b - a + TT - 1) / TT;
        if (slot < nt) {
            c.e = e;
            c.t0 = a + slot * TT;
            c.t_end = min(b, c.t0 + TT);
            return true;
        }
        slot -= nt;
    }
    return false;
}

// Equation 10 with 1/7.49 factored out: Y1 + Y2/14.98 + Y3/14.98^2 (+
// Y4/14.98^3 with four unfold steps).
constexpr float kR2 = static_cast<float>(1.0 / 14.98);
constexpr float kR3 = static_cast<float>(1.0 / (14.98 * 14.98));
constexpr float kR4 = static_cast<float>(1.0 / (14.98 * 14.98 * 14.98));
__device__ __forceinline__ constexpr float msd_plane_r(int p) { return p == 1 ? kR2 : (p == 2 ? kR3 : kR4); }

template <int VAR, int TT, int ST, int WST, int NCONV, int NEPI, int NISS, bool SEPI, bool DBG>
__global__ void __launch_bounds__(GemmCfg<VAR, TT, ST, WST, NCONV, NEPI, NISS, SEPI>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ GemmParams P)
{
    using C = GemmCfg<VAR, TT, ST, WST, NCONV, NEPI, NISS, SEPI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* wsm = smem + C::kBST * C::kStage;                         // weight slots
    float* red = reinterpret_cast<float*>(wsm + WST * C::kWSlot);      // split-K partials pushed by the cluster
    float* rr_part = reinterpret_cast<float*>(wsm + WST * C::kWSlot + C::kRedBytes);   // [NEPI-1][TT][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + WST * C::kWSlot + C::kRedBytes + C::kRRBytes);
    uint64_t* bfull_bar = bars;                 // [kBST] activation tile landed
    uint64_t* bfree_bar = bfull_bar + C::kBST;  // [kBST] activation stage free again (MMA done)
    uint64_t* sfree_bar = bfree_bar + C::kBST;  // [ST] operand stage free again (MMA done)
    uint64_t* afull_bar = sfree_bar + ST;       // [ST] A operand written to Tensor Memory
    uint64_t* wfull_bar = afull_bar + ST;       // [WST] weight slot landed
    uint64_t* wempty_bar = wfull_bar + WST;     // [WST] weight slot read by its converter group
    uint64_t* accfull_bar = wempty_bar + WST;        // [kNBuf] accumulator ready for the epilogue
    uint64_t* accempty_bar = accfull_bar + C::kNBuf; // [kNBuf] group accumulator read (and reset) by the epilogue
    uint64_t* done_bar = accempty_bar + C::kNBuf;    // [kMaxIssuers] all MMAs of an issuer completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + C::kMaxIssuers);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // A_max ring, one per epilogue warp: [4 * NEPI][2][TT] floats read as
    // float4: round up to a 16-byte boundary (the barriers before it end on
    // an 8-byte boundary only)
    float* amax_sm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(tmem_slot + 4) + 15) & ~uintptr_t(15));

    TileCoord tc;
    if (!resolve_tile(P, TT, tc)) return;          // uniform across the CTA

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int issuers = P.issuers;

    // K-chunk range of this split (split units keep groups whole).
    const int units = (P.kchunks + P.unit - 1) / P.unit;
    const int kc0 = min(P.kchunks, (tc.split * units / P.splits) * P.unit);
    const int kc1 = min(P.kchunks, ((tc.split + 1) * units / P.splits) * P.unit);
    const int nchunks = kc1 - kc0;
    const int n0 = tc.n_tile * kBN;
    const int grp0 = (kc0 * kKC) / P.g;                 // first group of this split

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kBST; ++s) {
            mbar_init(smem_addr(&bfull_bar[s]), 1);
            mbar_init(smem_addr(&bfree_bar[s]), 1);
        }
        for (int s = 0; s < ST; ++s) {
            mbar_init(smem_addr(&sfree_bar[s]), 1);
            mbar_init(smem_addr(&afull_bar[s]), 4);
        }
        for (int w = 0; w < WST; ++w) {
            mbar_init(smem_addr(&wfull_bar[w]), 1);
            mbar_init(smem_addr(&wempty_bar[w]), 4);
        }
        for (int b = 0; b < C::kNBuf; ++b) {
            mbar_init(smem_addr(&accfull_bar[b]), 1);
            mbar_init(smem_addr(&accempty_bar[b]), C::kEpiRR ? 4 : 4 * NEPI);
        }
        for (int q = 0; q < C::kMaxIssuers; ++q) mbar_init(smem_addr(&done_bar[q]), 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensor_map(&tmap);
    }
    if (warp == 1) tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The next kernel in the stream may start launching now; it waits
    // (griddep_wait) before touching anything this one writes.
    if (threadIdx.x == 0) griddep_launch_dependents();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_a0 = tmem + C::kAccCols;               // A operand stages
    const uint64_t tmo = P.timeout_ns;

    if (warp == 0 || warp == 1) {
        // ============================ producers ============================
        // Warp 0 streams the packed weights (and the scale rows when the
        // converter applies them) into the weight ring: constant inputs,
        // fetched without waiting for the previous kernel.  Warp 1 brings the
        // activation tiles (x, or the expansion kernel's A_int) into the
        // operand stages once that kernel has finished.  The whole warp runs
        // the loop (converged); lane 0 issues.
        const bool weights = warp == 0;
        if (nchunks > 0) {
            const uint8_t* wsrc = P.w[tc.e] + (static_cast<size_t>(tc.n_tile) * P.kchunks + kc0) * kWStage;
            const __half* ssrc = P.scale[tc.e];
            const uint32_t srow_bytes = static_cast<uint32_t>(min(kBN, P.N - n0)) * 2u;
            if (!weights) griddep_wait();
            const int ring = weights ? WST : C::kBST;
            uint64_t* fullb = weights ? wfull_bar : bfull_bar;
            // with one activation stage per operand stage the MMA's stage
            // commit frees both
            uint64_t* freeb = weights ? wempty_bar : (C::kBST == ST ? sfree_bar : bfree_bar);
            int issued = 0;
            // groups of gsz chunks: one copy into gsz consecutive slots (the
            // ring is a multiple of gsz: a group never wraps), completing on
            // the group's first slot's barrier; a short last group still
            // lands a whole box (past the end: zero fill or chunks nobody
            // reads), so every slot of it is waited free
            const int gsz = weights ? C::kWG : (TT == 16 ? P.bgroup : 1);
            if (gsz > 1) {
                int groups = 0;
                for (int i0 = 0; i0 < nchunks; i0 += gsz) {
                    const int nc = min(gsz, nchunks - i0);
                    const int s0 = i0 % ring;
                    const uint32_t ph = (i0 / ring) & 1;
                    bool free_ok = true;
                    for (int c = 0; c < gsz && free_ok; ++c)
                        free_ok = mbar_wait(smem_addr(&freeb[s0 + c]), ph ^ 1, tmo, P.status, abort_flag);
                    if (!free_ok) break;
                    if (lane == 0) {
                        const uint32_t fb = smem_addr(&fullb[s0]);
                        const int kc = kc0 + i0;
                        if (weights) {
                            mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nc) * kWStage);
                            bulk_g2s(smem_addr(wsm + s0 * C::kWSlot), wsrc + static_cast<size_t>(i0) * kWStage,
                                     static_cast<uint32_t>(nc) * kWStage, fb);
                        } else {
                            mbar_arrive_expect_tx(fb, static_cast<uint32_t>(gsz) * C::kBBytes);
                            if (C::kIsMsd) tma_load_4d(smem_addr(smem + s0 * C::kStage), &tmap, 0, tc.t0, 0, kc, fb);
                            else tma_load_3d(smem_addr(smem + s0 * C::kStage), &tmap, 0, tc.t0, 2 * kc, fb);
                        }
                    }
                    __syncwarp();
                    ++groups;
                }
                // Drain: the last group issued on each first slot has landed.
                const int gpr = ring / gsz;        // groups per ring cycle
                for (int k0 = 0; k0 < gpr && k0 < groups; ++k0) {
                    const int kl = k0 + ((groups - 1 - k0) / gpr) * gpr;
                    mbar_wait(smem_addr(&fullb[k0 * gsz]), ((kl * gsz) / ring) & 1, tmo, P.status, nullptr);
                }
            }
            for (int i = 0; i < nchunks && gsz == 1; ++i) {
                const int s = i % ring;
                const uint32_t ph = (i / ring) & 1;
                if (!mbar_wait(smem_addr(&freeb[s]), ph ^ 1, tmo, P.status, abort_flag)) break;
                if (lane == 0) {
                    const uint32_t fb = smem_addr(&fullb[s]);
                    const int kc = kc0 + i;
                    if (weights) {
                        uint8_t* ws = wsm + s * C::kWSlot;
                        int srows = 0, sgrp0 = 0;
                        if (C::kSBytes > 0) {
                            sgrp0 = (kc * kKC) / P.g;
                            srows = (P.g >= kKC) ? 1 : min(kKC / P.g, P.G - sgrp0);
                        }
                        mbar_arrive_expect_tx(fb, kWStage + srows * srow_bytes);
                        bulk_g2s(smem_addr(ws), wsrc + static_cast<size_t>(i) * kWStage, kWStage, fb);
                        for (int h = 0; h < srows; ++h)
                            bulk_g2s(smem_addr(ws + kWStage + h * 256), ssrc + static_cast<size_t>(sgrp0 + h) * P.N + n0,
                                     srow_bytes, fb);
                    } else {
                        uint8_t* st = smem + s * C::kStage;
                        mbar_arrive_expect_tx(fb, C::kBBytes);
                        if (C::kIsMsd) {
#pragma unroll
                            for (int r = 0; r < C::kVals; ++r)
                                tma_load_2d(smem_addr(st + r * TT * 128), &tmap, kc * kKC, r * P.M + tc.t0, fb);
                        } else {
                            tma_load_2d(smem_addr(st), &tmap, kc * kKC, tc.t0, fb);
                            tma_load_2d(smem_addr(st + TT * 128), &tmap, kc * kKC + 64, tc.t0, fb);
                        }
                    }
                }
                __syncwarp();
                ++issued;
            }
            // Drain: every copy issued has landed before the CTA may exit.
            for (int s = 0; s < ring && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / ring) * ring;
                mbar_wait(smem_addr(&fullb[s]), (last / ring) & 1, tmo, P.status, nullptr);
            }
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 2 + C::kMaxIssuers) {
        // ============================ MMA issuers ============================
        // Issuer q takes chunks q, q + issuers, ...; it waits for the chunk's
        // A operand (converter) and activation tile (producer), and one commit
        // per chunk frees the operand stage for both.  The warp runs
        // converged; lane 0 issues the MMAs and commits.
        const int q = warp - 2;
        // One lane runs the issuer's whole loop (waits, MMAs, commits): a warp
        // that reconverges after every MMA roughly doubles the issue cost of
        // each one.
        if (q < issuers && lane == 0) {
            // dequant: a tile's MMAs cover only its tokens, rounded up to the
            // MMA's N step of 16 (the ragged last tile of an expert segment
            // then costs a fraction of a full one); the rows past them are
            // never read back.  MSD stacks its digit planes along N: full N.
            const int n_eff = C::kIsMsd ? C::kMmaN : min(C::kMmaN, ((tc.t_end - tc.t0 + 15) / 16) * 16);
            const uint32_t idesc = C::kIsMsd ? idesc_s8_s32(C::kMmaN)
                                             : (C::kBf16 ? idesc_bf16_f32(n_eff) : idesc_f16_f32(n_eff));
            constexpr int kSteps = C::kIsMsd ? 4 : 8;         // MMA K steps per 128-deep chunk
            constexpr int kStepK = kKC / kSteps;
            // group bookkeeping without divisions in the step loop: K steps
            // per group (g is a multiple of 32, so of kStepK), as a shift when
            // it is a power of two
            const int gsteps = P.g / kStepK;
            const bool gpow2 = (gsteps & (gsteps - 1)) == 0;
            const int gshift = __ffs(gsteps) - 1;
            bool first_chunk = true;
            for (int i = q; i < nchunks; i += issuers) {
                const int s = i % ST;
                const uint32_t ph = (i / ST) & 1;
                const int bs = i % C::kBST;
                const uint32_t bph = (i / C::kBST) & 1;
                if (!mbar_wait(smem_addr(&afull_bar[s]), ph, tmo, P.status, abort_flag)) break;
                // (grouped activation copies, decode tile only, complete on
                // the group's first slot)
                const int bfs = TT == 16 ? bs - bs % P.bgroup : bs;
                if (!mbar_wait(smem_addr(&bfull_bar[bfs]), bph, tmo, P.status, abort_flag)) break;
                tc_fence_after();
                const uint64_t bdesc = smem_desc_sw128(smem_addr(smem + bs * C::kStage));
                const uint32_t a_base = tmem_a0 + s * C::kACols;
                const int kc = kc0 + i;
                const int nsteps = min(kSteps, (P.K - kc * kKC) / kStepK);   // K-padding steps are skipped
                const int step0 = i * kSteps;        // K step index from the split's first group boundary
                bool failed = false;
                if (C::kGroupAcc && gsteps == kSteps && nsteps == kSteps) {
                    // a group is exactly this chunk (g = 128): buffer i % NBUF,
                    // every step's operands and flags known at compile time
                    const int ab = i % C::kNBuf;
                    if (!mbar_wait(smem_addr(&accempty_bar[ab]), (i / C::kNBuf) & 1, tmo, P.status, abort_flag))
                        break;
                    tc_fence_after();
                    const uint32_t d = tmem + ab * C::kAccStride;
#pragma unroll
                    for (int j = 0; j < kSteps; ++j) {
                        const uint64_t bd =
                            C::kIsMsd ? bdesc + 2 * j : bdesc + ((j >> 2) * (TT * 128) >> 4) + 2 * (j & 3);
                        if (C::kIsMsd) mma_i8_ts(d, a_base + 8 * j, bd, idesc, j == 0 ? 0u : 1u);
                        else mma_f16_ts(d, a_base + 8 * j, bd, idesc, j == 0 ? 0u : 1u);
                    }
                    tc_commit(smem_addr(&accfull_bar[ab]));
                    tc_commit(smem_addr(&sfree_bar[s]));
                    if (C::kBST != ST) tc_commit(smem_addr(&bfree_bar[bs]));
                    first_chunk = false;
                    continue;
                }
                if (!C::kGroupAcc && nsteps == kSteps) {
                    // a full chunk into the issuer's one accumulator: every
                    // step's operands and flags known at compile time (the
                    // issuing lane's loop is on the tensor pipe's critical path)
                    const uint32_t d = tmem + q * C::kAccStride;
#pragma unroll
                    for (int j = 0; j < kSteps; ++j) {
                        const uint64_t bd = C::kIsMsd ? bdesc + 2 * j : bdesc + ((j >> 2) * (TT * 128) >> 4) + 2 * (j & 3);
                        mma_f16_ts(d, a_base + 8 * j, bd, idesc, (j == 0 && first_chunk) ? 0u : 1u);
                    }
                    tc_commit(smem_addr(&sfree_bar[s]));
                    if (C::kBST != ST) tc_commit(smem_addr(&bfree_bar[bs]));
                    first_chunk = false;
                    continue;
                }
#pragma unroll
                for (int j = 0; j < kSteps; ++j) {
                    if (j >= nsteps) break;
                    // B operand: 32-byte K steps inside the 128-byte swizzle row;
                    // DEQUANT's chunk spans two 64-wide atoms of TT rows each
                    const uint64_t bd = C::kIsMsd ? bdesc + 2 * j : bdesc + ((j >> 2) * (TT * 128) >> 4) + 2 * (j & 3);
                    if (C::kGroupAcc) {
                        const int st_ = step0 + j;
                        const int grel = gpow2 ? (st_ >> gshift) : (st_ / gsteps);     // group within the split
                        const int gpos = st_ - grel * gsteps;                          // step within the group
                        const int ab = grel % C::kNBuf;
                        if (gpos == 0) {
                            // the epilogue has read this buffer
                            if (!mbar_wait(smem_addr(&accempty_bar[ab]), (grel / C::kNBuf) & 1, tmo, P.status,
                                           abort_flag)) {
                                failed = true;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint32_t d = tmem + ab * C::kAccStride;
                        // a group's first K step overwrites the buffer
                        if (C::kIsMsd) mma_i8_ts(d, a_base + 8 * j, bd, idesc, gpos == 0 ? 0u : 1u);
                        else mma_f16_ts(d, a_base + 8 * j, bd, idesc, gpos == 0 ? 0u : 1u);
                        if (gpos == gsteps - 1) tc_commit(smem_addr(&accfull_bar[ab]));
                    } else {
                        mma_f16_ts(tmem + q * C::kAccStride, a_base + 8 * j, bd, idesc,
                                   (first_chunk && j == 0) ? 0u : 1u);
                    }
                }
                tc_commit(smem_addr(&sfree_bar[s]));
                if (C::kBST != ST) tc_commit(smem_addr(&bfree_bar[bs]));
                first_chunk = false;
                if (failed) break;
            }
            if (!C::kGroupAcc) tc_commit(smem_addr(&accfull_bar[q]));
            // Every MMA issued has completed before Tensor Memory is freed.
            tc_commit(smem_addr(&done_bar[q]));
            mbar_wait(smem_addr(&done_bar[q]), 0, tmo, P.status, nullptr);
        }
        __syncwarp();
    } else if (warp >= C::kConvWarp0 && warp < C::kEpiWarp0) {
        // ============================ converters ============================
        // Group cg takes chunks cg, cg + NCONV, ...: packed weights from the
        // weight ring -> registers -> the MMA A operand in Tensor Memory.
        const int cg = (warp - C::kConvWarp0) >> 2;            // converter group
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32);
        const int r = lane_base + lane;                        // weight row in the tile
        for (int i = cg; i < nchunks; i += NCONV) {
            const int s = i % ST;
            const uint32_t ph = (i / ST) & 1;
            const int w = i % WST;
            const uint32_t wph = (i / WST) & 1;
            // the slot's copy completes on its group's first slot's barrier
            if (!mbar_wait(smem_addr(&wfull_bar[w - w % C::kWG]), wph, tmo, P.status, abort_flag)) break;
            const uint8_t* wst = wsm + w * C::kWSlot;
            uint4 q[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) q[p] = *reinterpret_cast<const uint4*>(wst + p * 2048 + r * 16);
            __half sv[4];
            if (!C::kIsMsd && !SEPI) {
                const __half* sst = reinterpret_cast<const __half*>(wst + kWStage);
                const int kc = kc0 + i;
                const int sgrp0 = (kc * kKC) / P.g;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int row = (P.g >= kKC) ? 0 : ((kc * kKC + 32 * p) / P.g - sgrp0);
                    sv[p] = sst[row * kBN + r];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&wempty_bar[w]));      // weight slot read
            // the A operand columns of stage s are free once the MMA of the
            // stage's previous chunk has completed
            if (!mbar_wait(smem_addr(&sfree_bar[s]), ph ^ 1, tmo, P.status, abort_flag)) break;
            tc_fence_after();
            const uint32_t a_addr = tmem_a0 + s * C::kACols + (lane_base << 16);
            if (C::kIsMsd) {
W4A16_ROLE_UNROLL
                for (int p = 0; p < 4; ++p) {
                    uint32_t o[8];
                    int8_word(q[p].x, o + 0);
                    int8_word(q[p].y, o + 2);
                    int8_word(q[p].z, o + 4);
                    int8_word(q[p].w, o + 6);
                    tmem_st8(a_addr + 8 * p, o);
                }
            } else if (SEPI) {
W4A16_ROLE_UNROLL
                for (int p = 0; p < 4; ++p) {
                    uint32_t o[16];
                    if constexpr (C::kBf16) {
                        int4_to_bf162x4(q[p].x, o + 0);
                        int4_to_bf162x4(q[p].y, o + 4);
                        int4_to_bf162x4(q[p].z, o + 8);
                        int4_to_bf162x4(q[p].w, o + 12);
                    } else {
                        int4_to_half2x4(q[p].x, o + 0);
                        int4_to_half2x4(q[p].y, o + 4);
                        int4_to_half2x4(q[p].z, o + 8);
                        int4_to_half2x4(q[p].w, o + 12);
                    }
                    tmem_st16(a_addr + 16 * p, o);
                }
            } else {
W4A16_ROLE_UNROLL
                for (int p = 0; p < 4; ++p) {
                    const __half2 s2 = __halves2half2(sv[p], sv[p]);
                    uint32_t o[16];
                    int4_to_half2x4_scaled(q[p].x, s2, o + 0);
                    int4_to_half2x4_scaled(q[p].y, s2, o + 4);
                    int4_to_half2x4_scaled(q[p].z, s2, o + 8);
                    int4_to_half2x4_scaled(q[p].w, s2, o + 12);
                    tmem_st16(a_addr + 16 * p, o);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&afull_bar[s]));
        }
    } else if (warp >= C::kEpiWarp0) {
        // ============================ epilogue ============================
        const int eg = (warp - C::kEpiWarp0) >> 2;             // epilogue group
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32);
        const int r = lane_base + lane;
        const int n = n0 + r;
        const bool n_ok = n < P.N;
        const int nt = tc.t_end - tc.t0;
        constexpr int TE = C::kTokPerEpi;
        const int tb = C::kEpiRR ? 0 : eg * TE;                 // first token of this group
        const uint32_t t_addr = tmem + (lane_base << 16);
        // routed form (one expert per token): the tile's row -> (token, gate
        // weight) map, staged once per warp in the warp's own A_max ring (not
        // in use by then) so that the stores do not chase two dependent global
        // loads per element: [TT] tokens, then [TT] weights
        auto stage_map = [&]() {
            float* mp = amax_sm + (warp - C::kEpiWarp0) * 2 * TT;
            __syncwarp();
            for (int t = lane; t < TT; t += 32) {
                int d = -1;
                float wv = 0.f;
                if (t < nt) {
                    d = __ldg(P.row_dst + tc.t0 + t);
                    if (d >= 0) wv = __ldg(P.row_w + d);
                }
                mp[t] = __int_as_float(d);
                mp[TT + t] = wv;
            }
            __syncwarp();
        };
        // token t of the tile, column n, through the staged map
        auto store_mapped = [&](int t, float v) {
            const float* mp = amax_sm + (warp - C::kEpiWarp0) * 2 * TT;
            const int d = __float_as_int(mp[t]);
            if (d >= 0) store_elem<C::kBf16>(P.y + static_cast<size_t>(d) * P.N + n, v * mp[TT + t]);
        };
        float acc[TE];
#pragma unroll
        for (int t = 0; t < TE; ++t) acc[t] = 0.f;
        bool ok = true;

        if (C::kGroupAcc) {
            __syncwarp();
            if (lane == 0)          // release every buffer (this group's, round-robin) to the MMA
                for (int b = 0; b < C::kNBuf; ++b)
                    if (!C::kEpiRR || b % NEPI == eg) mbar_arrive(smem_addr(&accempty_bar[b]));
            griddep_wait();    // A_max comes from the expansion kernel; y is shared with earlier kernels

            const int ngroups = min(kc1 * kKC, P.K) / P.g - grp0;
            const __half* sc_e = P.scale[tc.e];
            const int jstep = C::kEpiRR ? NEPI : 1, j0 = C::kEpiRR ? eg : 0;
            // A_max of the tile's TT tokens for the next group, lane l holding
            // tokens l, l + 32, ...; each warp keeps its own two-slot ring in
            // shared memory, so only the warp synchronises
            constexpr int AMV = (TT + 31) / 32;
            float am_next[AMV];
            float sc_next = 0.f;
#pragma unroll
            for (int v = 0; v < AMV; ++v) {
                const int tok = lane + 32 * v;
                am_next[v] = (C::kIsMsd && j0 < ngroups && tok < nt)
                                 ? __ldg(P.amax + static_cast<size_t>(grp0 + j0) * P.M + tc.t0 + tok) : 0.f;
            }
            if (j0 < ngroups && n_ok && sc_e) sc_next = load_elem<C::kBf16>(sc_e + static_cast<size_t>(grp0 + j0) * P.N + n);
            float* am_ring = amax_sm + (warp - C::kEpiWarp0) * 2 * TT;
            for (int j = j0, jj = 0; j < ngroups; j += jstep, ++jj) {
                const int grp = grp0 + j;
                const int ab = j % C::kNBuf;
                const uint32_t abph = (j / C::kNBuf) & 1;
                float* am_slot = am_ring + (jj & 1) * TT;
                if (C::kIsMsd) {
#pragma unroll
                    for (int v = 0; v < AMV; ++v)
                        if (lane + 32 * v < TT) am_slot[lane + 32 * v] = am_next[v];
                }
                const float sc = sc_next;
                if (j + jstep < ngroups) {       // prefetch the next group's A_max and scale
                    if (C::kIsMsd) {
#pragma unroll
                        for (int v = 0; v < AMV; ++v) {
                            const int tok = lane + 32 * v;
                            am_next[v] =
                                tok < nt ? __ldg(P.amax + static_cast<size_t>(grp + jstep) * P.M + tc.t0 + tok) : 0.f;
                        }
                    }
                    if (n_ok && sc_e) sc_next = load_elem<C::kBf16>(sc_e + static_cast<size_t>(grp + jstep) * P.N + n);
                }
                if (C::kIsMsd) __syncwarp();
                if (ok && !mbar_wait(smem_addr(&accfull_bar[ab]), abph, tmo, P.status, abort_flag)) ok = false;
                if (!ok) continue;
                tc_fence_after();
                const uint32_t b_addr = t_addr + ab * C::kAccStride + tb;
                bool released = false;
                if (C::kIsMsd) {
                    const float scc = sc * kC1;
                    // equations 10-11 for 8 tokens of this column, and the
                    // debug window's copy of their Y_i and A_max
                    auto combine8 = [&](int c, const uint32_t (&yv)[C::kVals][8]) {
                        const float4 a0 = reinterpret_cast<const float4*>(am_slot + tb + 8 * c)[0];
                        const float4 a1 = reinterpret_cast<const float4*>(am_slot + tb + 8 * c)[1];
                        const float am[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                        for (int qq = 0; qq < 8; qq += 2) {
                            float2 v = make_float2(__int2float_rn(static_cast<int>(yv[0][qq])),
                                                   __int2float_rn(static_cast<int>(yv[0][qq + 1])));
#pragma unroll
                            for (int p = 1; p < C::kVals; ++p)
                                v = ffma2(make_float2(__int2float_rn(static_cast<int>(yv[p][qq])),
                                                      __int2float_rn(static_cast<int>(yv[p][qq + 1]))),
                                          make_float2(msd_plane_r(p), msd_plane_r(p)), v);
                            const float2 f = fmul2(make_float2(am[qq], am[qq + 1]), make_float2(scc, scc));
                            const float2 a = ffma2(v, f, make_float2(acc[8 * c + qq], acc[8 * c + qq + 1]));
                            acc[8 * c + qq] = a.x;
                            acc[8 * c + qq + 1] = a.y;
                        }
                        if (DBG && n_ok && n >= P.dbg_n0 && n < P.dbg_n1) {
                            const int wn = P.dbg_n1 - P.dbg_n0, wm = P.dbg_m1 - P.dbg_m0;
                            const size_t plane = static_cast<size_t>(wm) * P.G * wn;
#pragma unroll
                            for (int qq = 0; qq < 8; ++qq) {
                                const int t = tb + 8 * c + qq;
                                const int m = tc.t0 + t;
                                if (t < nt && m >= P.dbg_m0 && m < P.dbg_m1) {
                                    const size_t o = (static_cast<size_t>(m - P.dbg_m0) * P.G + grp) * wn + (n - P.dbg_n0);
#pragma unroll
                                    for (int p = 0; p < C::kVals; ++p)
                                        P.dbg_yint[p * plane + o] = static_cast<int32_t>(yv[p][qq]);
                                    if (n == P.dbg_n0)
                                        P.dbg_amax[static_cast<size_t>(m - P.dbg_m0) * P.G + grp] = am[qq];
                                }
                            }
                        }
                    };
                    if constexpr (C::kEpiBurst) {
                        // all of the group's sums into registers at once, then
                        // the buffer goes back to the MMA before the combine:
                        // the next group's MMAs run without this warp's
                        // Tensor Memory reads beside them
                        uint32_t yv[TE / 8][C::kVals][8];
#pragma unroll
                        for (int c = 0; c < TE / 8; ++c)
#pragma unroll
                            for (int p = 0; p < C::kVals; ++p) tmem_ld8(b_addr + p * TT + 8 * c, yv[c][p]);
                        tmem_ld_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_addr(&accempty_bar[ab]));
                        released = true;
#pragma unroll
                        for (int c = 0; c < TE / 8; ++c) combine8(c, yv[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < TE / 8; ++c) {
                            uint32_t yv[C::kVals][8];   // Y1..YS of 8 tokens
#pragma unroll
                            for (int p = 0; p < C::kVals; ++p) tmem_ld8(b_addr + p * TT + 8 * c, yv[p]);
                            tmem_ld_wait();
                            combine8(c, yv);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < TE / 16; ++c) {
                        uint32_t v[16];
                        tmem_ld16(b_addr + 16 * c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; ++k) acc[16 * c + k] = fmaf(__uint_as_float(v[k]), sc, acc[16 * c + k]);
                    }
                }
                if (!released) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&accempty_bar[ab]));
                }
            }
            if (C::kEpiRR) {
                // groups 1..NEPI-1 hand their partial sums to group 0, which
                // adds them in group order (deterministic)
                if (eg > 0)
#pragma unroll
                    for (int t = 0; t < TE; ++t) rr_part[((eg - 1) * TT + t) * kBN + r] = acc[t];
                named_bar_sync(1 + NEPI, C::kEpiThreads);
                if (eg == 0)
                    for (int e2 = 1; e2 < NEPI; ++e2)
#pragma unroll
                        for (int t = 0; t < TE; ++t) acc[t] += rr_part[((e2 - 1) * TT + t) * kBN + r];
            }
            if (P.row_dst != nullptr) {
                stage_map();
                if (ok && P.write_y && n_ok)
                    for (int t = 0; t < TE; ++t)
                        if (tb + t < nt) store_mapped(tb + t, acc[t]);
            } else if (ok && P.splits == 1 && P.write_y && n_ok && (!C::kEpiRR || eg == 0)) {
#pragma unroll
                for (int t = 0; t < TE; ++t)
                    if (tb + t < nt) store_elem<C::kBf16>(P.y + static_cast<size_t>(tc.t0 + tb + t) * P.N + n, acc[t]);
            }
        } else {
            // one accumulator over all of K per issuer (scales applied by the
            // converter); issuers with no chunk left theirs unwritten
            griddep_wait();
            if (P.row_dst != nullptr) stage_map();
            const int nacc = min(issuers, nchunks);
            ok = nchunks > 0;
            for (int q = 0; q < nacc && ok; ++q)
                ok = mbar_wait(smem_addr(&accfull_bar[q]), 0, tmo, P.status, abort_flag);
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < TE / 16; ++c) {
                    float v[16];
                    {
                        uint32_t u[16];
                        tmem_ld16(t_addr + tb + 16 * c, u);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(u[k]);
                    }
                    for (int q = 1; q < nacc; ++q) {
                        uint32_t u[16];
                        tmem_ld16(t_addr + q * C::kAccStride + tb + 16 * c, u);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; ++k) v[k] += __uint_as_float(u[k]);
                    }
                    // the routed/dense choice is made once per chunk of 16
                    // tokens, outside the unrolled stores: the dense path
                    // runs plain stores only
                    if (P.write_y && n_ok) {
                        if (P.row_dst == nullptr) {
                            __half* yp = P.y + static_cast<size_t>(tc.t0 + tb + 16 * c) * P.N + n;
                            const int kmax = nt - (tb + 16 * c);
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                if (k < kmax) store_elem<C::kBf16>(yp + static_cast<size_t>(k) * P.N, v[k]);
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                if (tb + 16 * c + k < nt) store_mapped(tb + 16 * c + k, v[k]);
                        }
                    }
                }
                tc_fence_before();
            }
        }

        // Split-K (decode tile only): push this CTA's partial sums into the
        // reduction buffer of the cluster rank that owns them: element
        // e = t * 128 + r belongs to rank e / per and lands in slot
        // [this rank][e - owner * per] there.
        if (C::kRedBytes > 0 && P.splits > 1 && ok && (!C::kEpiRR || eg == 0)) {
            const int S = P.splits;
            const int per = (TT * kBN + S - 1) / S;
            const uint32_t me = cluster_ctarank();
            const uint32_t red_base = smem_addr(red);
#pragma unroll
            for (int t = 0; t < TE; ++t) {
                const int e = (tb + t) * kBN + r;
                const int owner = e / per;
                st_cluster_f32(map_to_rank(red_base + 4u * static_cast<uint32_t>(me * per + (e - owner * per)),
                                           static_cast<uint32_t>(owner)),
                               acc[t]);
            }
        }
    }

    // Split-K: one cluster barrier (every thread of every CTA) makes all
    // pushed partials visible; each rank then adds, in rank order
    // (deterministic), the S partials of the elements it owns and stores y.
    // After the barrier no CTA touches another's shared memory.
    if (C::kRedBytes > 0 && P.splits > 1) {
        __syncwarp();
        cluster_sync_all();
        if (warp >= C::kEpiWarp0 && P.write_y && !*abort_flag) {
            const int S = P.splits;
            const int per = (TT * kBN + S - 1) / S;
            const int me = static_cast<int>(cluster_ctarank());
            const int nt = tc.t_end - tc.t0;
            for (int el = threadIdx.x - 32 * C::kEpiWarp0; el < per; el += C::kEpiThreads) {
                const int e = me * per + el;
                const int t = e / kBN;
                const int nn = n0 + (e % kBN);
                if (t >= nt || nn >= P.N) continue;
                float sum = 0.f;
                for (int sp = 0; sp < S; ++sp) sum += red[sp * per + el];
                store_row<C::kBf16>(P, tc.t0 + t, nn, sum);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// A wait on a barrier that nothing completes: exercises the bounded-wait
// path (status word set, kernel returns) without hanging the device.
__global__ void selftest_wait_kernel(uint32_t* status, unsigned long long timeout_ns)
{
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, timeout_ns, status, nullptr);
}

}  // namespace w4a16
