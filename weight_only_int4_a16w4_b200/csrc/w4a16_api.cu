// w4a16_api.cu -- host side of libw4a16.so: argument validation, workspace
// layout, TMA descriptors, launch-shape choice and the extern "C" entry
// points declared in include/w4a16.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/w4a16.h"
#include "w4a16_gemv.cuh"
#include "w4a16_gemv_mma.cuh"
#include "w4a16_kernels.cuh"
#include "w4a16_moe.cuh"

using namespace w4a16;


namespace {

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};

constexpr size_t kHeaderBytes = 256;   // device status word + padding
constexpr int kMaxSmemOptin = 227 * 1024;   // dynamic shared memory a CTA may opt in to

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
int cdiv(int a, int b) { return (a + b - 1) / b; }

bool is_msd_op(int op) { return op == W4A16_OP_MSD || op == W4A16_OP_MSD_2STEP || op == W4A16_OP_MSD_4STEP; }
bool op_ok(int op) { return is_msd_op(op) || op == W4A16_OP_DEQUANT || op == W4A16_OP_DEQUANT_BF16; }
// MSD digit planes of an op (the unfold steps)
int op_steps(int op) { return op == W4A16_OP_MSD_2STEP ? 2 : (op == W4A16_OP_MSD_4STEP ? 4 : 3); }

bool group_ok(int g)
{
    if (g <= 0 || g % 32) return false;
    return (g <= kKC) ? (kKC % g == 0) : (g % kKC == 0);
}

// ---------------------------------------------------------------- device facts

// cudaFuncSetAttribute acts on the current device, so a kernel's attributes
// are set once per (kernel instance, device); each launcher keeps one of
// these.  `init` runs with the device current and returns its CUDA status.
struct PerDeviceInit {
    std::mutex mu;
    std::atomic<bool> done[64] = {};
    cudaError_t err[64] = {};
    template <typename Fn>
    cudaError_t get(Fn&& init)
    {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (done[dev].load(std::memory_order_acquire)) return err[dev];
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev].load(std::memory_order_relaxed)) {
            err[dev] = init();
            done[dev].store(true, std::memory_order_release);
        }
        return err[dev];
    }
};

int sm_count()
{
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cached[dev] = v;
    }
    return cached[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D K-major tensor map, 128-byte swizzle, box = (box_k, box_rows).
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, int K, int rows,
              int box_k, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * elem_bytes};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_k), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// element type of the activation tiles of a dequant call
CUtensorMapDataType act_dtype(int op)
{
    return op == W4A16_OP_DEQUANT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// The decode tile's activations, kBCopyGroup chunks per box (dense calls with
// K % 128 == 0).  MSD: the digit planes [S][M][K] int8 seen as dims (128 k
// of a chunk, row, plane, chunk); dequant: x [M][K] 16-bit as (64 k of a
// half-chunk, row, half-chunk).  A box lands as kBCopyGroup consecutive
// operand stages, each laid out as the two-dimensional boxes lay one out.
bool make_map_grouped(CUtensorMap* map, const void* base, int op, int M, int K, int box_rows)
{
    auto fn = encode_fn();
    if (!fn || K % kKC != 0) return false;
    CUresult r;
    if (is_msd_op(op)) {
        const int S = op_steps(op);
        cuuint64_t dims[4] = {static_cast<cuuint64_t>(kKC), static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(K / kKC)};
        cuuint64_t strides[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M) * K,
                                 static_cast<cuuint64_t>(kKC)};
        cuuint32_t box[4] = {static_cast<cuuint32_t>(kKC), static_cast<cuuint32_t>(box_rows),
                             static_cast<cuuint32_t>(S), static_cast<cuuint32_t>(kBCopyGroup)};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(K / 64)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, 128};
        cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(2 * kBCopyGroup)};
        cuuint32_t estr[3] = {1, 1, 1};
        r = fn(map, act_dtype(op), 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- launch shapes

struct Shape {
    int TT;
    int splits;
    int unit;
    int t_slots;
    int n_tiles;
    int kchunks;
};

bool small_tile(int op, int M) { (void)op; return M <= 16; }

// Tokens per tile.  Dequant: 256 (MMA N = 256: each MMA carries ~136 cycles
// of tensor work, well above its issue cost -- measured 1014 vs 786 TFLOP/s
// at M = N = K = 4096) while that still gives at least two CTAs per SM,
// else 128 (grouped calls: T rows).
// bf16 dequant: 128 (its per-group accumulators take two 128-column
// buffers of Tensor Memory; 256 tokens would not fit beside the operand).
int tile_tokens(int op, int M, int N)
{
    if (small_tile(op, M)) return 16;
    // MSD: 64 tokens (2 or 3 planes), 32 with four planes (4 x 32 MMA rows
    // keep two per-group accumulator buffers within Tensor Memory)
    if (is_msd_op(op)) return op_steps(op) == 4 ? 32 : 64;
    if (op == W4A16_OP_DEQUANT_BF16) return 128;
    return static_cast<long long>(cdiv(M, 256)) * cdiv(N, kBN) >= 2ll * sm_count() ? 256 : 128;
}

// Split-K factor for a decode-sized dense call: the CTAs of one column tile
// split K among themselves and reduce through distributed shared memory
// (a cluster of `splits` CTAs).  At most one CTA per SM, so that the next
// kernel in the stream can already occupy the second slot (programmatic
// dependent launch); the largest factor that keeps all CTAs in one wave.
int choose_splits(int tiles, int units)
{
    const int sms = sm_count();
    if (tiles >= sms || units <= 1) return 1;
    int best = 1;
    for (int s = 2; s <= std::min(units, 8); ++s)
        if (static_cast<long>(tiles) * s <= sms) best = s;
    return best;
}

Shape dense_shape(int op, int M, int K, int N, int g)
{
    Shape s;
    s.TT = tile_tokens(op, M, N);
    s.kchunks = cdiv(K, kKC);
    s.n_tiles = cdiv(N, kBN);
    s.t_slots = std::max(1, cdiv(M, s.TT));
    s.unit = std::max(1, g / kKC);
    const int units = cdiv(s.kchunks, s.unit);
    s.splits = small_tile(op, M) ? choose_splits(s.n_tiles * s.t_slots, units) : 1;
    return s;
}

Shape grouped_shape(int op, int T, int K, int N, int g, int E)
{
    Shape s;
    s.TT = tile_tokens(op, std::max(T, 17), N);   // grouped calls never use the decode tile
    s.kchunks = cdiv(K, kKC);
    s.n_tiles = cdiv(N, kBN);
    s.t_slots = std::max(1, cdiv(T, s.TT) + E);
    s.unit = std::max(1, g / kKC);
    s.splits = 1;
    return s;
}

// ---------------------------------------------------------------- the CUDA-core decode GEMV

// the warp-MMA GEMV's rows: S digit planes x MR tokens must fit 8 MMA rows
int gemv_mma_max_m(int op) { return is_msd_op(op) ? 8 / op_steps(op) : 8; }

// rows of the instance: 1, 2, 4 or 8 tokens, capped by the variant
int gemv_mma_rows(int op, int M)
{
    const int r = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
    const int cap = is_msd_op(op) ? (op_steps(op) == 2 ? 4 : 2) : 8;
    return std::min(r, cap);
}

template <int VAR, int NW>
int gemv_mma_smem_nw(int MR, int M, int np, int ppg)
{
    // instances exist for S * MR <= 8 only
    constexpr int S = is_msd(VAR) ? msd_steps(VAR) : 1;
    switch (MR) {
        case 1: return MgCfg<VAR, 1, NW>::smem_bytes(M, np, ppg);
        case 2: return MgCfg<VAR, 2, NW>::smem_bytes(M, np, ppg);
        case 4: return MgCfg<VAR, 4 * S <= 8 ? 4 : 1, NW>::smem_bytes(M, np, ppg);
        default: return MgCfg<VAR, 8 * S <= 8 ? 8 : 1, NW>::smem_bytes(M, np, ppg);
    }
}

template <int VAR>
int gemv_mma_smem_var(int MR, int NW, int M, int np, int ppg)
{
    return NW == 32 ? gemv_mma_smem_nw<VAR, 32>(MR, M, np, ppg) : gemv_mma_smem_nw<VAR, 16>(MR, M, np, ppg);
}

int gemv_mma_smem_nw_op(int op, int NW, int M, int K, int g)
{
    const int np = K / 32, ppg = g / 32, MR = gemv_mma_rows(op, M);
    switch (op) {
        case W4A16_OP_MSD: return gemv_mma_smem_var<kMsd>(MR, NW, M, np, ppg);
        case W4A16_OP_MSD_2STEP: return gemv_mma_smem_var<kMsd2>(MR, NW, M, np, ppg);
        case W4A16_OP_MSD_4STEP: return gemv_mma_smem_var<kMsd4>(MR, NW, M, np, ppg);
        default: return gemv_mma_smem_var<kDeq>(MR, NW, M, np, ppg);
    }
}

// Warps per CTA of the warp-MMA GEMV.  Measured on B200 (us per call, 16 vs
// 32 warps): dequant at M <= 2 with N >= 8192 gains from 32 warps of one
// quad-round each (K 4096, N 14336: 17.3 -> 16.3; K = N = 8192: 18.2 ->
// 16.8); at N = 4096 and for MSD, 16 warps are as fast or faster (MSD
// K 4096, N 14336: 14.7 vs 15.6); 8 warps lose everywhere.
int gemv_mma_warps(int op, int M, int K, int N, int g)
{
    int nw = 16;
    if (!is_msd_op(op) && M <= 2 && N >= 8192) nw = 32;
    if (nw == 32 && gemv_mma_smem_nw_op(op, 32, M, K, g) > kMaxSmemOptin) nw = 16;
    return nw;
}

int gemv_mma_smem(int op, int M, int K, int N, int g)
{
    return gemv_mma_smem_nw_op(op, gemv_mma_warps(op, M, K, N, g), M, K, g);
}

// The kernel of a dense call with a handful of rows.  Measured on B200
// (consecutive dependent calls, weights streamed from HBM):
//  * g % 128 == 0, M <= 8 (dequant) or M <= 2 (MSD): the warp-MMA GEMV
//    (w4a16_gemv_mma.cuh) beats the CUDA-core GEMV and the tensor-core
//    decode tile at every size measured;
//  * other g (32, 64) and M <= 4: the CUDA-core GEMV (w4a16_gemv.cuh), as the
//    tensor tile is weak there (fp16 only: bf16 takes the decode tile);
//  * everything else: the tensor-core decode tile.
enum SmallKernel { kSmallNone = 0, kSmallCuda = 1, kSmallMma = 2 };

int small_kernel(int op, int M, int K, int N, int g, int E)
{
    if (E != 1 || M < 1) return kSmallNone;
    const bool mma_ok = g % 128 == 0 && M <= gemv_mma_max_m(op) &&
                        static_cast<long long>(N / 8) * sm_count() < (1ll << 31) &&
                        gemv_mma_smem(op, M, K, N, g) <= kMaxSmemOptin;
    // (the CUDA-core GEMV is built for fp16 dequant and three-step MSD only)
    const bool cuda_ok = (op == W4A16_OP_DEQUANT || op == W4A16_OP_MSD) && M <= 4 &&
                         static_cast<long long>(M) * K <= kGemvMaxMK;
    if (mma_ok) return kSmallMma;
    if (cuda_ok && g % 128 != 0) return kSmallCuda;
    return kSmallNone;
}

// CTAs of a GEMV: one per SM at most, never more than there are column
// blocks.
int gemv_ctas(int nblk) { return std::min(nblk, sm_count()); }

struct WsLayout {
    size_t xq = 0, amax = 0, rec = 0, total = 0;
};

WsLayout ws_layout(int op, const Shape& s, int M, int K, int N, int g, int E = 1)
{
    (void)s;
    (void)N;
    WsLayout L;
    size_t off = kHeaderBytes;
    if (is_msd_op(op)) {
        const int S = op_steps(op);
        L.xq = off;
        off += align256(static_cast<size_t>(S) * M * K);
        L.amax = off;
        off += align256(static_cast<size_t>(K / g) * M * 4);
        if (small_kernel(op, M, K, N, g, E) != kSmallNone) {
            // the decode GEMV's digit records [K/32][M][gemv_rec_words(S)]
            L.rec = off;
            off += align256(static_cast<size_t>(K / 32) * M * gemv_rec_words(S) * 4);
        }
    }
    L.total = off;
    return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

w4a16_status check_shape(int M, int K, int N, int g)
{
    if (M < 0 || K <= 0 || N <= 0 || g <= 0) return W4A16_ERR_INVALID_ARG;
    if (N % 8 || K % g) return W4A16_ERR_INVALID_ARG;
    if (!group_ok(g)) return W4A16_ERR_UNSUPPORTED;
    return W4A16_OK;
}

// ---------------------------------------------------------------- kernel launch

template <int VAR, int TT, int ST, int WST, int NCONV, int NEPI, int NISS, bool SEPI, bool DBG = false>
w4a16_status launch_gemm(const CUtensorMap& map, const GemmParams& P, dim3 grid, cudaStream_t stream)
{
    using C = GemmCfg<VAR, TT, ST, WST, NCONV, NEPI, NISS, SEPI>;
    auto kern = gemm_kernel<VAR, TT, ST, WST, NCONV, NEPI, NISS, SEPI, DBG>;
    static PerDeviceInit kattr;
    const cudaError_t attr_err = kattr.get([&] {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        return e;
    });
    if (attr_err != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    // split-K reduces through the decode tile's own partial buffer
    if (P.splits > 1 && (C::kRedBytes == 0 || P.splits > 16)) return W4A16_ERR_UNSUPPORTED;
    if (P.issuers < 1 || P.issuers > NISS || ST % P.issuers != 0) return W4A16_ERR_UNSUPPORTED;
    if (C::kGroupAcc && P.issuers > 1 && P.g != kKC) return W4A16_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (P.splits > 1) {   // the split-K CTAs of one tile form a cluster (see gemm_kernel)
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = static_cast<unsigned>(P.splits);
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kern, map, P) != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    return W4A16_OK;
}

// Kernel instances (variant, token tile, operand stages, weight stages,
// converter groups, epilogue groups, MMA issuers, scale in the epilogue);
// one CTA per SM, 512 Tensor Memory columns.
//   decode (M <= 16): MSD <16, 8, 12, 2, 2, 4>   DEQUANT <16, 4, 12, 2, 2, 4, scale in epilogue>
//     four MMA issuers: each small MMA (N = 48 / 16) holds its issuing
//     thread for far longer than the tensor core needs (two issuers with
//     more operand stages measured 40 % slower); two epilogue groups take
//     alternate K groups; 16 activation stages of their own
//   larger M:         MSD <64, 4, 4, 1, 4, 1>   DEQUANT <128, 4, 4, 2, 1, 2>
//     MSD: four epilogue groups of 16 tokens, each reading all of a group's
//     sums before handing the buffer back (measured at prefill: 463 ->
//     452 us against two groups of 32 tokens), one converter group (the
//     warps that fit beside them); DEQUANT two issuers, each into its own
//     accumulator (<256, 2, 4, 2, 2, 1> when there are enough tiles)
//   bf16 dequant: <16, 4, 12, 2, 2, 4, scale in epilogue> and
//     <128, 4, 4, 2, 2, 2, scale in epilogue>
w4a16_status launch_for(int op, int TT, const CUtensorMap& map, const GemmParams& P, dim3 grid, cudaStream_t s)
{
    if (op == W4A16_OP_MSD) {
        // the Y_int debug window: the product instance's template parameters
        // with the window writes switched on
        if (P.dbg_yint != nullptr) {
            if (TT == 16) return launch_gemm<kMsd, 16, 8, 12, 2, 2, 4, false, true>(map, P, grid, s);
            return launch_gemm<kMsd, 64, 4, 4, 1, 4, 1, false, true>(map, P, grid, s);
        }
        if (TT == 16) return launch_gemm<kMsd, 16, 8, 12, 2, 2, 4, false>(map, P, grid, s);
        return launch_gemm<kMsd, 64, 4, 4, 1, 4, 1, false>(map, P, grid, s);
    }
    if (op == W4A16_OP_MSD_2STEP) {
        if (P.dbg_yint != nullptr) {
            if (TT == 16) return launch_gemm<kMsd2, 16, 8, 12, 2, 2, 4, false, true>(map, P, grid, s);
            return launch_gemm<kMsd2, 64, 4, 4, 1, 4, 1, false, true>(map, P, grid, s);
        }
        if (TT == 16) return launch_gemm<kMsd2, 16, 8, 12, 2, 2, 4, false>(map, P, grid, s);
        return launch_gemm<kMsd2, 64, 4, 4, 1, 4, 1, false>(map, P, grid, s);
    }
    if (op == W4A16_OP_MSD_4STEP) {
        // 4 x 16-row activation stages: 8 weight stages keep shared memory in bounds
        if (P.dbg_yint != nullptr) {
            if (TT == 16) return launch_gemm<kMsd4, 16, 8, 8, 2, 2, 4, false, true>(map, P, grid, s);
            return launch_gemm<kMsd4, 32, 4, 4, 2, 2, 1, false, true>(map, P, grid, s);
        }
        if (TT == 16) return launch_gemm<kMsd4, 16, 8, 8, 2, 2, 4, false>(map, P, grid, s);
        return launch_gemm<kMsd4, 32, 4, 4, 2, 2, 1, false>(map, P, grid, s);
    }
    if (op == W4A16_OP_DEQUANT_BF16) {
        if (TT == 16) return launch_gemm<kDeqBf16, 16, 4, 12, 2, 2, 4, true>(map, P, grid, s);
        return launch_gemm<kDeqBf16, 128, 4, 4, 2, 2, 2, true>(map, P, grid, s);
    }
    if (TT == 16) return launch_gemm<kDeq, 16, 4, 12, 2, 2, 4, true>(map, P, grid, s);
    if (TT == 256) return launch_gemm<kDeq, 256, 2, 4, 2, 2, 1, false>(map, P, grid, s);
    return launch_gemm<kDeq, 128, 4, 4, 2, 1, 2, false>(map, P, grid, s);
}

template <int VPL, int S>
cudaError_t launch_expand_vpl(int blocks, const __half* x, int M, int K, int g, int8_t* xq, float* amax,
                              cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expand_kernel<VPL, S>, x, M, K, g, xq, amax);
}

template <int S>
cudaError_t launch_expand_s(int blocks, const __half* xh, int M, int K, int g, int8_t* xq, float* amax,
                            cudaStream_t s)
{
    switch (g / 32) {
        case 1: return launch_expand_vpl<1, S>(blocks, xh, M, K, g, xq, amax, s);
        case 2: return launch_expand_vpl<2, S>(blocks, xh, M, K, g, xq, amax, s);
        case 4: return launch_expand_vpl<4, S>(blocks, xh, M, K, g, xq, amax, s);
        case 8: return launch_expand_vpl<8, S>(blocks, xh, M, K, g, xq, amax, s);
        case 12: return launch_expand_vpl<12, S>(blocks, xh, M, K, g, xq, amax, s);
        case 16: return launch_expand_vpl<16, S>(blocks, xh, M, K, g, xq, amax, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int S, int STEPS>
cudaError_t launch_expand8(const __half* x, int M, int K, int g, int8_t* xq, float* amax, cudaStream_t s)
{
    // warp tasks of STEPS * 256 values; at most 8 CTAs of 8 warps per SM,
    // the warps loop over the rest
    const long long tasks = (static_cast<long long>(M) * K / 8 + 32 * STEPS - 1) / (32 * STEPS);
    const int blocks = static_cast<int>(std::min<long long>((tasks + 7) / 8, 8ll * sm_count()));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    switch (g / 8) {
        case 4: return cudaLaunchKernelEx(&cfg, expand8_kernel<4, S, STEPS>, x, M, K, g, xq, amax);
        case 8: return cudaLaunchKernelEx(&cfg, expand8_kernel<8, S, STEPS>, x, M, K, g, xq, amax);
        case 16: return cudaLaunchKernelEx(&cfg, expand8_kernel<16, S, STEPS>, x, M, K, g, xq, amax);
        case 32: return cudaLaunchKernelEx(&cfg, expand8_kernel<32, S, STEPS>, x, M, K, g, xq, amax);
        default: return cudaErrorInvalidValue;
    }
}

// Four 256-value blocks per warp task once that still gives every SM 64
// warps' worth of tasks (large M: more loads in flight per warp); one block
// per task below that, where the warps' count matters more.
template <int S>
cudaError_t launch_expand8_s(const __half* x, int M, int K, int g, int8_t* xq, float* amax, cudaStream_t s)
{
    const long long tasks4 = (static_cast<long long>(M) * K / 8 + 127) / 128;
    if (tasks4 >= 64ll * sm_count()) return launch_expand8<S, 4>(x, M, K, g, xq, amax, s);
    return launch_expand8<S, 1>(x, M, K, g, xq, amax, s);
}

w4a16_status launch_expand(int op, const void* x, int M, int K, int g, int8_t* xq, float* amax, cudaStream_t s)
{
    const long long warps = static_cast<long long>(M) * (K / g);
    const int blocks = static_cast<int>((warps + 7) / 8);
    const __half* xh = static_cast<const __half*>(x);
    const int v = g / 32;
    if (!(v == 1 || v == 2 || v == 4 || v == 8 || v == 12 || v == 16)) return W4A16_ERR_UNSUPPORTED;
    cudaError_t e;
    if (g <= 256) {
        // groups of up to 256 values: the 16-byte-per-thread form
        switch (op_steps(op)) {
            case 2: e = launch_expand8_s<2>(xh, M, K, g, xq, amax, s); break;
            case 4: e = launch_expand8_s<4>(xh, M, K, g, xq, amax, s); break;
            default: e = launch_expand8_s<3>(xh, M, K, g, xq, amax, s); break;
        }
    } else {
        switch (op_steps(op)) {
            case 2: e = launch_expand_s<2>(blocks, xh, M, K, g, xq, amax, s); break;
            case 4: e = launch_expand_s<4>(blocks, xh, M, K, g, xq, amax, s); break;
            default: e = launch_expand_s<3>(blocks, xh, M, K, g, xq, amax, s); break;
        }
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    return W4A16_OK;
}

void base_params(GemmParams& P, int op, int M, int K, int N, int g, const Shape& s, void* ws)
{
    std::memset(&P, 0, sizeof(P));
    P.M = M;
    P.K = K;
    P.N = N;
    P.g = g;
    P.G = K / g;
    P.kchunks = s.kchunks;
    P.n_tiles = s.n_tiles;
    P.t_slots = s.t_slots;
    P.splits = s.splits;
    P.unit = s.unit;
    P.E = 1;
    // the large DEQUANT tile has one accumulator per MMA issuer (two); the
    // bf16 tile two issuers when a group is one chunk (each owns one of the
    // per-group buffers); the 256-token tile has one issuer
    P.issuers = (op == W4A16_OP_DEQUANT && s.TT == 128) ? 2 : 1;
    if (op == W4A16_OP_DEQUANT_BF16 && s.TT == 128) P.issuers = (g == kKC) ? 2 : 1;
    P.status = static_cast<uint32_t*>(ws);
    P.timeout_ns = g_timeout_ns.load();
    P.write_y = 1;
    P.bgroup = 1;
}

template <int VAR, int MR, bool DBG = false>
w4a16_status launch_gemv_mr(const GemvParams& P, cudaStream_t stream)
{
    using C = GemvCfg<VAR, MR>;
    auto kern = gemv_kernel<VAR, MR, DBG>;
    const int smem = C::smem_bytes(P.M, P.K);
    static PerDeviceInit kattr;
    const auto set_smem = [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemOptin);
    };
    if (kattr.get(set_smem) != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    if (smem > kMaxSmemOptin) return W4A16_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(P.ctas), 1, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, P) != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    return W4A16_OK;
}

template <int VAR, int MR, int NW, bool DBG = false>
w4a16_status launch_gemv_mma_nw(const GemvParams& P, cudaStream_t stream)
{
    auto kern = gemv_mma_kernel<VAR, MR, NW, DBG>;
    const int smem = MgCfg<VAR, MR, NW>::smem_bytes(P.M, P.K / 32, P.g / 32);
    static PerDeviceInit kattr;
    const auto set_smem = [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemOptin);
    };
    if (kattr.get(set_smem) != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    if (smem > kMaxSmemOptin) return W4A16_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(P.ctas), 1, 1);
    cfg.blockDim = dim3(NW * 32, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, P) != cudaSuccess) {
        (void)cudaGetLastError();
        return W4A16_ERR_CUDA;
    }
    return W4A16_OK;
}

template <int VAR, int MR, bool DBG = false>
w4a16_status launch_gemv_mma_mr(const GemvParams& P, cudaStream_t stream)
{
    const int op = VAR == kMsd ? W4A16_OP_MSD : VAR == kMsd2 ? W4A16_OP_MSD_2STEP
                 : VAR == kMsd4 ? W4A16_OP_MSD_4STEP : W4A16_OP_DEQUANT;
    if (gemv_mma_warps(op, P.M, P.K, P.N, P.g) == 32) return launch_gemv_mma_nw<VAR, MR, 32, DBG>(P, stream);
    return launch_gemv_mma_nw<VAR, MR, 16, DBG>(P, stream);
}

template <int NSUB, int S>
cudaError_t launch_gemv_expand_n(const __half* x, int M, int K, int g, uint32_t* rec, cudaStream_t s)
{
    const int span = NSUB * kKC;
    const long long warps = static_cast<long long>(M) * ((K + span - 1) / span);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((warps + 7) / 8), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_expand_kernel<NSUB, S>, x, M, K, g, rec);
}

template <int S>
cudaError_t launch_gemv_expand_s(const __half* x, int M, int K, int g, uint32_t* rec, cudaStream_t s)
{
    switch (std::max(1, g / kKC)) {
        case 1: return launch_gemv_expand_n<1, S>(x, M, K, g, rec, s);
        case 2: return launch_gemv_expand_n<2, S>(x, M, K, g, rec, s);
        case 3: return launch_gemv_expand_n<3, S>(x, M, K, g, rec, s);
        case 4: return launch_gemv_expand_n<4, S>(x, M, K, g, rec, s);
        default: return cudaErrorInvalidValue;
    }
}

// the warp-MMA GEMV of an MSD variant, MR chosen by M; DBG: the Y_int
// window instance
template <int VAR, bool DBG>
w4a16_status launch_gemv_mma_msd_dbg(const GemvParams& P, int op, cudaStream_t stream)
{
    switch (gemv_mma_rows(op, P.M)) {
        case 1: return launch_gemv_mma_mr<VAR, 1, DBG>(P, stream);
        case 2: return launch_gemv_mma_mr<VAR, 2, DBG>(P, stream);
        default:
            if constexpr (4 * msd_steps(VAR) <= 8) return launch_gemv_mma_mr<VAR, 4, DBG>(P, stream);
            return W4A16_ERR_UNSUPPORTED;
    }
}

template <int VAR>
w4a16_status launch_gemv_mma_msd(const GemvParams& P, int op, cudaStream_t stream)
{
    return P.dbg_yint != nullptr ? launch_gemv_mma_msd_dbg<VAR, true>(P, op, stream)
                                 : launch_gemv_mma_msd_dbg<VAR, false>(P, op, stream);
}

w4a16_status launch_gemv(int op, bool mma, const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                         int g, void* y, void* ws, const Shape& s, const WsLayout& L, cudaStream_t stream,
                         int32_t* dbg_yint = nullptr, float* dbg_amax = nullptr, int m0 = 0, int m1 = 0, int n0 = 0,
                         int n1 = 0)
{
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    GemvParams P;
    std::memset(&P, 0, sizeof(P));
    P.dbg_yint = dbg_yint;
    P.dbg_amax = dbg_amax;
    P.dbg_m0 = m0;
    P.dbg_m1 = m1;
    P.dbg_n0 = n0;
    P.dbg_n1 = n1;
    P.x = static_cast<const __half*>(x);
    P.w = static_cast<const uint8_t*>(w_packed);
    P.scale = static_cast<const __half*>(scale);
    P.y = static_cast<__half*>(y);
    P.M = M;
    P.K = K;
    P.N = N;
    P.g = g;
    P.G = K / g;
    P.kchunks = s.kchunks;
    P.npieces = K / 32;
    P.nblk = mma ? N / 8 : cdiv(N, 32);
    P.ctas = gemv_ctas(P.nblk);
    if (is_msd_op(op)) {
        uint32_t* rec = reinterpret_cast<uint32_t*>(wsb + L.rec);
        P.rec = rec;
        const __half* xh = static_cast<const __half*>(x);
        if (std::max(1, g / kKC) > 4) return W4A16_ERR_UNSUPPORTED;
        if (!mma && op != W4A16_OP_MSD) return W4A16_ERR_UNSUPPORTED;   // CUDA-core GEMV: three steps only
        cudaError_t e;
        switch (op_steps(op)) {
            case 2: e = launch_gemv_expand_s<2>(xh, M, K, g, rec, stream); break;
            case 4: e = launch_gemv_expand_s<4>(xh, M, K, g, rec, stream); break;
            default: e = launch_gemv_expand_s<3>(xh, M, K, g, rec, stream); break;
        }
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return W4A16_ERR_CUDA;
        }
        if (mma) {
            switch (op_steps(op)) {
                case 2: return launch_gemv_mma_msd<kMsd2>(P, op, stream);
                case 4: return launch_gemv_mma_msd<kMsd4>(P, op, stream);
                default: return launch_gemv_mma_msd<kMsd>(P, op, stream);
            }
        }
        if (P.dbg_yint != nullptr) {
            if (M == 1) return launch_gemv_mr<kMsd, 1, true>(P, stream);
            if (M == 2) return launch_gemv_mr<kMsd, 2, true>(P, stream);
            return launch_gemv_mr<kMsd, 4, true>(P, stream);
        }
        if (M == 1) return launch_gemv_mr<kMsd, 1>(P, stream);
        if (M == 2) return launch_gemv_mr<kMsd, 2>(P, stream);
        return launch_gemv_mr<kMsd, 4>(P, stream);
    }
    if (op == W4A16_OP_DEQUANT_BF16) {
        if (!mma) return W4A16_ERR_UNSUPPORTED;   // small_kernel never picks the CUDA-core GEMV for bf16
        switch (gemv_mma_rows(op, M)) {
            case 1: return launch_gemv_mma_mr<kDeqBf16, 1>(P, stream);
            case 2: return launch_gemv_mma_mr<kDeqBf16, 2>(P, stream);
            case 4: return launch_gemv_mma_mr<kDeqBf16, 4>(P, stream);
            default: return launch_gemv_mma_mr<kDeqBf16, 8>(P, stream);
        }
    }
    if (mma) {
        switch (gemv_mma_rows(op, M)) {
            case 1: return launch_gemv_mma_mr<kDeq, 1>(P, stream);
            case 2: return launch_gemv_mma_mr<kDeq, 2>(P, stream);
            case 4: return launch_gemv_mma_mr<kDeq, 4>(P, stream);
            default: return launch_gemv_mma_mr<kDeq, 8>(P, stream);
        }
    }
    if (M == 1) return launch_gemv_mr<kDeq, 1>(P, stream);
    if (M == 2) return launch_gemv_mr<kDeq, 2>(P, stream);
    return launch_gemv_mr<kDeq, 4>(P, stream);
}

// Shared body of the dense MSD / DEQUANT calls and the debug window.
w4a16_status dense_matmul(int op, const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                          int g, void* y, void* ws, size_t ws_bytes, cudaStream_t stream, int32_t* dbg_yint,
                          float* dbg_amax, int m0, int m1, int n0, int n1)
{
    w4a16_status st = check_shape(M, K, N, g);
    if (st != W4A16_OK) return st;
    if (is_msd_op(op) && g > kMaxGroupMsd) return W4A16_ERR_UNSUPPORTED;
    if (M == 0) return W4A16_OK;
    const bool debug = dbg_yint != nullptr;
    if (!x || !w_packed || (!scale && !debug) || (!y && !debug) || !ws) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_packed) || (scale && !aligned16(scale)) || (y && !aligned16(y)) ||
        !aligned16(ws))
        return W4A16_ERR_INVALID_ARG;
    const Shape s = dense_shape(op, M, K, N, g);
    const WsLayout L = ws_layout(op, s, M, K, N, g);
    if (ws_bytes < L.total) return W4A16_ERR_WORKSPACE;

    GemmParams P;
    base_params(P, op, M, K, N, g, s, ws);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    P.w[0] = static_cast<const uint8_t*>(w_packed);
    P.scale[0] = static_cast<const __half*>(scale);
    P.y = static_cast<__half*>(y);
    if (debug) {
        P.write_y = 0;
        P.dbg_yint = dbg_yint;
        P.dbg_amax = dbg_amax;
        P.dbg_m0 = m0;
        P.dbg_m1 = m1;
        P.dbg_n0 = n0;
        P.dbg_n1 = n1;
    }
    // the debug window runs the very kernels (and launch shapes) of the
    // product call, in instances that write Y_int instead of y; the GEMV adds
    // parts of a group into it, so it starts at zero
    if (debug) {
        const size_t wbytes = static_cast<size_t>(op_steps(op)) * (m1 - m0) * (K / g) * (n1 - n0) * sizeof(int32_t);
        if (cudaMemsetAsync(dbg_yint, 0, wbytes, stream) != cudaSuccess) return W4A16_ERR_CUDA;
    }
    {
        const int sk = small_kernel(op, M, K, N, g, 1);
        if (sk != kSmallNone)
            return launch_gemv(op, sk == kSmallMma, x, w_packed, scale, M, K, N, g, y, ws, s, L, stream, dbg_yint,
                               dbg_amax, m0, m1, n0, n1);
    }
    CUtensorMap map;
    if (is_msd_op(op)) {
        int8_t* xq = reinterpret_cast<int8_t*>(wsb + L.xq);
        float* amax = reinterpret_cast<float*>(wsb + L.amax);
        st = launch_expand(op, x, M, K, g, xq, amax, stream);
        if (st != W4A16_OK) return st;
        P.amax = amax;
        if (s.TT == 16 && make_map_grouped(&map, xq, op, M, K, s.TT)) P.bgroup = kBCopyGroup;
        else if (!make_map(&map, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, op_steps(op) * M, kKC, s.TT))
            return W4A16_ERR_CUDA;
    } else {
        if (s.TT == 16 && make_map_grouped(&map, x, op, M, K, s.TT)) P.bgroup = kBCopyGroup;
        else if (!make_map(&map, x, act_dtype(op), 2, K, M, 64, s.TT)) return W4A16_ERR_CUDA;
    }
    // four MMA issuers on the decode tile when a group is exactly one
    // 128-deep chunk: each issuer then owns one of the per-group
    // accumulator buffers
    if (s.TT == 16) P.issuers = (g == kKC) ? 4 : 1;
    dim3 grid(s.n_tiles, s.splits, s.t_slots);
    return launch_for(op, s.TT, map, P, grid, stream);
}

}  // namespace

// Scratch of w4a16_msd_matmul_noalloc: one array in device memory per GPU
// that loads the library.  Host code must not use the symbol itself as an
// address; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[W4A16_NOALLOC_SCRATCH_BYTES];

namespace {

// The driver's cuCtxGetCurrent, reached through the runtime (the library
// does not link the driver library itself).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of g_noalloc_scratch on the current device, looked up with
// that device current the first time it is needed in the current context and
// kept per device together with the context it belongs to: a call in
// another context (a device reset re-creates the primary context and may
// load the module elsewhere) looks the address up again.  nullptr on failure.
void* noalloc_scratch()
{
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    static CUcontext owner[64] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    const CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return nullptr;
    CUcontext ctx = nullptr;   // null while the runtime has not bound a context yet
    if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (ctx == nullptr || addr[dev] == nullptr || owner[dev] != ctx) {
        void* p = nullptr;
        // (binds the device's primary context if none is current yet)
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return nullptr;
        }
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
        addr[dev] = p;
        owner[dev] = ctx;
    }
    return addr[dev];
}

}  // namespace

// =================================================================== C ABI

extern "C" {

const char* w4a16_status_string(w4a16_status s)
{
    switch (s) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_INVALID_ARG: return "invalid argument";
        case W4A16_ERR_UNSUPPORTED: return "unsupported shape or group size";
        case W4A16_ERR_WORKSPACE: return "workspace missing or too small";
        case W4A16_ERR_CUDA: return "CUDA error";
        case W4A16_ERR_TIMEOUT: return "device wait timed out";
        case W4A16_ERR_BAD_INDEX: return "device-side index out of range";
    }
    return "unknown status";
}

size_t w4a16_packed_bytes(int K, int N)
{
    if (K <= 0 || N <= 0) return 0;
    return static_cast<size_t>(cdiv(N, kBN)) * cdiv(K, kKC) * kWStage;
}

w4a16_status w4a16_workspace_size(int op, int M, int K, int N, int group_size, int E, size_t* bytes)
{
    if (!bytes) return W4A16_ERR_INVALID_ARG;
    if (!op_ok(op)) return W4A16_ERR_INVALID_ARG;
    if (E < 1 || E > kMaxExperts) return W4A16_ERR_INVALID_ARG;
    w4a16_status st = check_shape(M, K, N, group_size);
    if (st != W4A16_OK) return st;
    if (is_msd_op(op) && group_size > kMaxGroupMsd) return W4A16_ERR_UNSUPPORTED;
    const Shape s = (E == 1) ? dense_shape(op, M, K, N, group_size) : grouped_shape(op, M, K, N, group_size, E);
    *bytes = ws_layout(op, s, M, K, N, group_size, E).total;
    return W4A16_OK;
}

w4a16_status w4a16_repack(const uint8_t* w_logical, int K, int N, void* w_packed, w4a16_stream_t stream)
{
    if (!w_logical || !w_packed || K <= 0 || N <= 0 || (K & 1) || (N % 8)) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(w_packed)) return W4A16_ERR_INVALID_ARG;
    const int kchunks = cdiv(K, kKC), n_tiles = cdiv(N, kBN);
    const long long total = static_cast<long long>(n_tiles) * kchunks * 2048;
    const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 65535LL * 8));
    repack_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        w_logical, K, N, kchunks, n_tiles, static_cast<uint32_t*>(w_packed));
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

w4a16_status w4a16_msd_matmul(const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                              int group_size, void* y, void* workspace, size_t workspace_bytes,
                              w4a16_stream_t stream)
{
    return dense_matmul(W4A16_OP_MSD, x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, 0, 0, 0, 0);
}

w4a16_status w4a16_dequant_matmul(const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                                  int group_size, void* y, void* workspace, size_t workspace_bytes,
                                  w4a16_stream_t stream)
{
    return dense_matmul(W4A16_OP_DEQUANT, x, w_packed, scale, M, K, N, group_size, y, workspace,
                        workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, 0, 0, 0, 0);
}

w4a16_status w4a16_dequant_matmul_bf16(const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                                       int group_size, void* y, void* workspace, size_t workspace_bytes,
                                       w4a16_stream_t stream)
{
    return dense_matmul(W4A16_OP_DEQUANT_BF16, x, w_packed, scale, M, K, N, group_size, y, workspace,
                        workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, 0, 0, 0, 0);
}

namespace {
int steps_op(int steps)
{
    return steps == 2 ? W4A16_OP_MSD_2STEP : steps == 3 ? W4A16_OP_MSD : steps == 4 ? W4A16_OP_MSD_4STEP : -1;
}
}  // namespace

w4a16_status w4a16_msd_matmul_steps(int steps, const void* x, const void* w_packed, const void* scale, int M, int K,
                                    int N, int group_size, void* y, void* workspace, size_t workspace_bytes,
                                    w4a16_stream_t stream)
{
    const int op = steps_op(steps);
    if (op < 0) return W4A16_ERR_INVALID_ARG;
    return dense_matmul(op, x, w_packed, scale, M, K, N, group_size, y, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, 0, 0, 0, 0);
}

w4a16_status w4a16_msd_debug_yint_steps(int steps, const void* x, const void* w_packed, int M, int K, int N,
                                        int group_size, int m0, int m1, int n0, int n1, int32_t* yint, float* amax,
                                        void* workspace, size_t workspace_bytes, w4a16_stream_t stream)
{
    const int op = steps_op(steps);
    if (op < 0 || !yint || !amax) return W4A16_ERR_INVALID_ARG;
    if (m0 < 0 || m1 <= m0 || m1 > M || n0 < 0 || n1 <= n0 || n1 > N) return W4A16_ERR_INVALID_ARG;
    // equation 9 needs no scale
    return dense_matmul(op, x, w_packed, nullptr, M, K, N, group_size, nullptr, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream), yint, amax, m0, m1, n0, n1);
}

w4a16_status w4a16_msd_debug_yint(const void* x, const void* w_packed, int M, int K, int N, int group_size,
                                  int m0, int m1, int n0, int n1, int32_t* yint, float* amax, void* workspace,
                                  size_t workspace_bytes, w4a16_stream_t stream)
{
    return w4a16_msd_debug_yint_steps(3, x, w_packed, M, K, N, group_size, m0, m1, n0, n1, yint, amax, workspace,
                                      workspace_bytes, stream);
}

namespace {
// The grouped matmul; row_dst / row_w (routed form, one expert per token)
// store row r at y row row_dst[r] times row_w[row_dst[r]] (nullptr: row r).
w4a16_status grouped_impl(int op, const void* x, const void* const* w_packed, const void* const* scale,
                          const int32_t* offsets, int E, int T, int K, int N, int group_size, void* y,
                          void* workspace, size_t workspace_bytes, const int32_t* row_dst, const float* row_w,
                          w4a16_stream_t stream)
{
    if (!op_ok(op)) return W4A16_ERR_INVALID_ARG;
    if (E < 1 || E > kMaxExperts) return W4A16_ERR_INVALID_ARG;
    w4a16_status st = check_shape(T, K, N, group_size);
    if (st != W4A16_OK) return st;
    if (is_msd_op(op) && group_size > kMaxGroupMsd) return W4A16_ERR_UNSUPPORTED;
    if (T == 0) return W4A16_OK;
    if (!x || !w_packed || !scale || !offsets || !y || !workspace) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return W4A16_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
        if (!w_packed[e] || !scale[e] || !aligned16(w_packed[e]) || !aligned16(scale[e]))
            return W4A16_ERR_INVALID_ARG;
    const Shape s = grouped_shape(op, T, K, N, group_size, E);
    const WsLayout L = ws_layout(op, s, T, K, N, group_size, E);
    if (workspace_bytes < L.total) return W4A16_ERR_WORKSPACE;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    GemmParams P;
    base_params(P, op, T, K, N, group_size, s, workspace);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    P.E = E;
    P.offsets = offsets;
    for (int e = 0; e < E; ++e) {
        P.w[e] = static_cast<const uint8_t*>(w_packed[e]);
        P.scale[e] = static_cast<const __half*>(scale[e]);
    }
    P.y = static_cast<__half*>(y);
    P.row_dst = row_dst;
    P.row_w = row_w;
    CUtensorMap map;
    if (is_msd_op(op)) {
        int8_t* xq = reinterpret_cast<int8_t*>(wsb + L.xq);
        float* amax = reinterpret_cast<float*>(wsb + L.amax);
        st = launch_expand(op, x, T, K, group_size, xq, amax, cs);
        if (st != W4A16_OK) return st;
        P.amax = amax;
        if (!make_map(&map, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, op_steps(op) * T, kKC, s.TT))
            return W4A16_ERR_CUDA;
    } else {
        if (!make_map(&map, x, act_dtype(op), 2, K, T, 64, s.TT)) return W4A16_ERR_CUDA;
    }
    dim3 grid(s.n_tiles, 1, s.t_slots);
    return launch_for(op, s.TT, map, P, grid, cs);
}
}  // namespace

w4a16_status w4a16_grouped_matmul(int op, const void* x, const void* const* w_packed, const void* const* scale,
                                  const int32_t* offsets, int E, int T, int K, int N, int group_size, void* y,
                                  void* workspace, size_t workspace_bytes, w4a16_stream_t stream)
{
    return grouped_impl(op, x, w_packed, scale, offsets, E, T, K, N, group_size, y, workspace, workspace_bytes,
                        nullptr, nullptr, stream);
}

w4a16_status w4a16_moe_align(const int32_t* topk_ids, int T, int topk, int E, int32_t* offsets,
                             int32_t* sorted_token, int32_t* inv_pos, void* workspace, size_t workspace_bytes,
                             w4a16_stream_t stream)
{
    if (T < 0 || topk < 1 || E < 1 || E > kMoeMaxExperts) return W4A16_ERR_INVALID_ARG;
    if (static_cast<long long>(T) * topk >= (1ll << 31)) return W4A16_ERR_INVALID_ARG;
    if (!offsets || !workspace) return W4A16_ERR_INVALID_ARG;
    if (workspace_bytes < kHeaderBytes) return W4A16_ERR_WORKSPACE;
    if (T > 0 && (!topk_ids || !sorted_token || !inv_pos)) return W4A16_ERR_INVALID_ARG;
    moe_align_kernel<<<1, kMoeAlignThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        topk_ids, T * topk, topk, E, offsets, sorted_token, inv_pos, static_cast<uint32_t*>(workspace));
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

w4a16_status w4a16_moe_gather(const void* x, const int32_t* sorted_token, int rows, int K, void* x_sorted,
                              w4a16_stream_t stream)
{
    if (rows < 0 || K <= 0 || K % 8) return W4A16_ERR_INVALID_ARG;
    if (rows == 0) return W4A16_OK;
    if (!x || !sorted_token || !x_sorted || !aligned16(x) || !aligned16(x_sorted)) return W4A16_ERR_INVALID_ARG;
    moe_gather_kernel<<<cdiv(rows, 8), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(x), sorted_token, rows, K / 8, static_cast<uint4*>(x_sorted));
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

namespace {
w4a16_status moe_combine(bool bf16, const void* y_sorted, const int32_t* inv_pos, const float* topk_weights, int T,
                         int topk, int N, void* y, w4a16_stream_t stream)
{
    if (T < 0 || topk < 1 || N <= 0 || N % 8) return W4A16_ERR_INVALID_ARG;
    if (static_cast<long long>(T) * topk >= (1ll << 31)) return W4A16_ERR_INVALID_ARG;
    if (T == 0) return W4A16_OK;
    if (!y_sorted || !inv_pos || !topk_weights || !y || !aligned16(y_sorted) || !aligned16(y))
        return W4A16_ERR_INVALID_ARG;
    auto kern = bf16 ? moe_combine_kernel<true> : moe_combine_kernel<false>;
    kern<<<cdiv(T, 8), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const __half*>(y_sorted), inv_pos, topk_weights, T, topk, N, static_cast<__half*>(y));
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}
}  // namespace

w4a16_status w4a16_moe_combine(const void* y_sorted, const int32_t* inv_pos, const float* topk_weights, int T,
                               int topk, int N, void* y, w4a16_stream_t stream)
{
    return moe_combine(false, y_sorted, inv_pos, topk_weights, T, topk, N, y, stream);
}

w4a16_status w4a16_moe_combine_bf16(const void* y_sorted, const int32_t* inv_pos, const float* topk_weights, int T,
                                    int topk, int N, void* y, w4a16_stream_t stream)
{
    return moe_combine(true, y_sorted, inv_pos, topk_weights, T, topk, N, y, stream);
}

namespace {
struct MoeLayout {
    size_t grouped = 0, offsets = 0, sorted = 0, inv = 0, xs = 0, ys = 0, total = 0;
};

w4a16_status moe_layout(int op, int T, int topk, int K, int N, int g, int E, MoeLayout* L)
{
    if (T < 0 || topk < 1) return W4A16_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(T) * topk;
    if (rows >= (1ll << 31)) return W4A16_ERR_INVALID_ARG;
    size_t gws = 0;
    const w4a16_status st = w4a16_workspace_size(op, static_cast<int>(rows), K, N, g, E, &gws);
    if (st != W4A16_OK) return st;
    size_t off = align256(gws);
    L->grouped = gws;
    L->offsets = off;
    off += align256(static_cast<size_t>(E + 1) * 4);
    L->sorted = off;
    off += align256(static_cast<size_t>(rows) * 4);
    L->inv = off;
    off += align256(static_cast<size_t>(rows) * 4);
    L->xs = off;
    off += align256(static_cast<size_t>(rows) * K * 2);
    L->ys = off;
    off += align256(static_cast<size_t>(rows) * N * 2);
    L->total = off;
    return W4A16_OK;
}
}  // namespace

w4a16_status w4a16_moe_workspace_size(int op, int T, int topk, int K, int N, int group_size, int E, size_t* bytes)
{
    if (!bytes) return W4A16_ERR_INVALID_ARG;
    MoeLayout L;
    const w4a16_status st = moe_layout(op, T, topk, K, N, group_size, E, &L);
    if (st == W4A16_OK) *bytes = L.total;
    return st;
}

w4a16_status w4a16_moe_matmul(int op, const void* x, const int32_t* topk_ids, const float* topk_weights,
                              const void* const* w_packed, const void* const* scale, int E, int T, int topk, int K,
                              int N, int group_size, void* y, void* workspace, size_t workspace_bytes,
                              w4a16_stream_t stream)
{
    MoeLayout L;
    w4a16_status st = moe_layout(op, T, topk, K, N, group_size, E, &L);
    if (st != W4A16_OK) return st;
    if (T == 0) return W4A16_OK;
    if (!x || !topk_ids || !topk_weights || !y || !workspace) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return W4A16_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return W4A16_ERR_WORKSPACE;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    int32_t* offsets = reinterpret_cast<int32_t*>(wsb + L.offsets);
    int32_t* sorted = reinterpret_cast<int32_t*>(wsb + L.sorted);
    int32_t* inv = reinterpret_cast<int32_t*>(wsb + L.inv);
    const int rows = T * topk;
    // the grouped matmul's workspace comes first, so the status word at the
    // start of `workspace` is shared by every step
    if ((st = w4a16_moe_align(topk_ids, T, topk, E, offsets, sorted, inv, workspace, L.grouped, stream)) != W4A16_OK)
        return st;
    if ((st = w4a16_moe_gather(x, sorted, rows, K, wsb + L.xs, stream)) != W4A16_OK) return st;
    if (topk == 1) {
        // one expert per token: the matmul stores each row at its token, times
        // the gate weight (the un-permute fused into its stores); tokens whose
        // id took no row get zeros
        if ((st = grouped_impl(op, wsb + L.xs, w_packed, scale, offsets, E, rows, K, N, group_size, y, workspace,
                               L.grouped, sorted, topk_weights, stream)) != W4A16_OK)
            return st;
        moe_zero_unrouted_kernel<<<cdiv(T, 8), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
            inv, T, N / 8, static_cast<uint4*>(y));
        return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
    }
    if ((st = w4a16_grouped_matmul(op, wsb + L.xs, w_packed, scale, offsets, E, rows, K, N, group_size, wsb + L.ys,
                                   workspace, L.grouped, stream)) != W4A16_OK)
        return st;
    return moe_combine(op == W4A16_OP_DEQUANT_BF16, wsb + L.ys, inv, topk_weights, T, topk, N, y, stream);
}

w4a16_status w4a16_msd_matmul_noalloc(const void* x, const void* w_packed, const void* scale, int M, int K, int N,
                                      int group_size, void* y, w4a16_stream_t stream)
{
    size_t need = 0;
    w4a16_status st = w4a16_workspace_size(W4A16_OP_MSD, M, K, N, group_size, 1, &need);
    if (st != W4A16_OK) return st;
    if (need > W4A16_NOALLOC_SCRATCH_BYTES) return W4A16_ERR_WORKSPACE;
    if (M == 0) return W4A16_OK;
    void* ws = noalloc_scratch();
    if (ws == nullptr) return W4A16_ERR_CUDA;
    // the status word must start at zero
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, kHeaderBytes, cs) != cudaSuccess) return W4A16_ERR_CUDA;
    return w4a16_msd_matmul(x, w_packed, scale, M, K, N, group_size, y, ws, W4A16_NOALLOC_SCRATCH_BYTES, stream);
}

w4a16_status w4a16_read_status(const void* workspace, w4a16_stream_t stream, uint32_t* status)
{
    if (!workspace || !status) return W4A16_ERR_INVALID_ARG;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return W4A16_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return W4A16_ERR_CUDA;
    if (*status & W4A16_DEVICE_TIMEOUT) return W4A16_ERR_TIMEOUT;
    return (*status & W4A16_DEVICE_BAD_EXPERT) ? W4A16_ERR_BAD_INDEX : W4A16_OK;
}

void w4a16_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns); }

w4a16_status w4a16_selftest_wait_timeout(void* workspace, uint64_t timeout_ns, w4a16_stream_t stream)
{
    if (!workspace || !aligned16(workspace)) return W4A16_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace),
                                                                             timeout_ns);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // extern "C"
