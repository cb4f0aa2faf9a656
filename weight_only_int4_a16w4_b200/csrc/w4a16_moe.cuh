// w4a16_moe.cuh -- routing prep of the grouped (mixture-of-experts) form.
//
// The grouped matmul takes each expert's tokens as one contiguous segment of
// rows (offsets[E+1]); a router hands over topk_ids [T][topk] (token t's
// j-th expert) and gate weights.  The mixture-of-experts scheduling of the
// Humming article (aihirek.info, MoE section) and the moe_align_block_size
// step of the FlagGems operator list (pwwt.cn) start from exactly that.
// Three kernels:
//
//  * moe_align_kernel: a stable grouping of the entries i = t*topk + j by
//    expert (increasing i within an expert): offsets, the token of every
//    sorted row and every entry's row.  One CTA of 32 warps; warp w owns a
//    contiguous run of entries, counts its experts with __match_any_sync (one
//    leader per expert per 32 entries), the per-(warp, expert) counts are
//    turned into row bases by a scan over (expert, warp), and a second walk
//    places each entry at base + (its rank among equal experts before it in
//    the same 32).  The result is unique, so it is compared bit for bit.  An
//    id outside [0, E) takes no row and sets W4A16_DEVICE_BAD_EXPERT.
//  * moe_gather_kernel: x rows into sorted order (a warp per row, 16-byte
//    loads, four in flight per lane); rows without an entry are zero.
//  * moe_combine_kernel: y[t] = sum_j w[t][j] * y_sorted[row of (t, j)], fp32
//    sums in increasing j, fp16 out (a warp per token, four 16-byte loads in
//    flight per lane); the bf16 instance reads and writes bf16.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace w4a16 {

constexpr int kMoeAlignThreads = 1024;
constexpr int kMoeAlignWarps = kMoeAlignThreads / 32;
constexpr int kMoeMaxExperts = 64;
constexpr uint32_t kDeviceBadExpert = 2u;   // status bit (W4A16_DEVICE_BAD_EXPERT)

__global__ void __launch_bounds__(kMoeAlignThreads) moe_align_kernel(const int32_t* __restrict__ ids, int n, int topk,
                                                                     int E, int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ sorted_token,
                                                                     int32_t* __restrict__ inv_pos,
                                                                     uint32_t* __restrict__ status)
{
    __shared__ int cnt[kMoeAlignWarps][kMoeMaxExperts];   // counts, then running row bases
    __shared__ int off_s[kMoeMaxExperts + 1];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = static_cast<int>((static_cast<long long>(warp) * n) / kMoeAlignWarps);
    const int c1 = static_cast<int>((static_cast<long long>(warp + 1) * n) / kMoeAlignWarps);
    for (int e = lane; e < kMoeMaxExperts; e += 32) cnt[warp][e] = 0;
    __syncwarp();

    auto key_of = [&](int i) {
        if (i >= c1) return -1;
        const int e = ids[i];
        return (e >= 0 && e < E) ? e : -1;
    };

    // counts per (warp, expert)
    for (int base = c0; base < c1; base += 32) {
        const int key = key_of(base + lane);
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) cnt[warp][key] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();

    // offsets[e] = entries of the experts below e; then cnt[w][e] = the row
    // of warp w's first entry of expert e
    if (tid < E) {
        int tot = 0;
        for (int w = 0; w < kMoeAlignWarps; ++w) tot += cnt[w][tid];
        off_s[tid + 1] = tot;
    }
    __syncthreads();
    if (tid == 0) {
        off_s[0] = 0;
        for (int e = 0; e < E; ++e) off_s[e + 1] += off_s[e];
    }
    __syncthreads();
    if (tid <= E) offsets[tid] = off_s[tid];
    if (tid < E) {
        int run = off_s[tid];
        for (int w = 0; w < kMoeAlignWarps; ++w) {
            const int c = cnt[w][tid];
            cnt[w][tid] = run;
            run += c;
        }
    }
    __syncthreads();

    // place every entry
    const unsigned below = (1u << lane) - 1u;
    for (int base = c0; base < c1; base += 32) {
        const int i = base + lane;
        const int key = key_of(i);
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0) {
            const int pos = cnt[warp][key] + __popc(peers & below);
            sorted_token[pos] = i / topk;
            inv_pos[i] = pos;
        } else if (i < c1) {
            inv_pos[i] = -1;
            atomicOr(status, kDeviceBadExpert);
        }
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) cnt[warp][key] += __popc(peers);
        __syncwarp();
    }
    // rows no entry took
    for (int p = off_s[E] + tid; p < n; p += kMoeAlignThreads) sorted_token[p] = -1;
}

// x_sorted[r] = x[sorted_token[r]] (zero where sorted_token[r] < 0); kv =
// K / 8 16-byte vectors per row; a warp per row, four loads in flight per
// lane.
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint4* __restrict__ x,
                                                         const int32_t* __restrict__ sorted_token, int rows, int kv,
                                                         uint4* __restrict__ x_sorted)
{
    constexpr int U = 4;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int src = sorted_token[row];
    uint4* dst = x_sorted + static_cast<size_t>(row) * kv;
    if (src < 0) {
        for (int v = lane; v < kv; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    const uint4* s = x + static_cast<size_t>(src) * kv;
    for (int v0 = lane; v0 < kv; v0 += 32 * U) {
        uint4 t[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (v0 + 32 * u < kv) t[u] = s[v0 + 32 * u];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (v0 + 32 * u < kv) dst[v0 + 32 * u] = t[u];
    }
}

// y[t][c .. c+7] = sum_j w[t][j] * y_sorted[inv_pos[t*topk+j]][c .. c+7],
// fp32 sums in increasing j (entries without a row skipped), a warp per
// token; each lane keeps four 16-byte loads in flight (columns c, c + 256,
// c + 512, c + 768).  BF: y_sorted and y hold bf16 bit patterns.
template <bool BF>
__global__ void __launch_bounds__(256) moe_combine_kernel(const __half* __restrict__ y_sorted,
                                                          const int32_t* __restrict__ inv_pos,
                                                          const float* __restrict__ weights, int T, int topk, int N,
                                                          __half* __restrict__ y)
{
    constexpr int U = 4;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    for (int c0 = lane * 8; c0 < N; c0 += 256 * U) {
        float acc[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[u][q] = 0.f;
        for (int j = 0; j < topk; ++j) {
            const int pos = inv_pos[t * topk + j];
            if (pos < 0) continue;
            const float wj = weights[t * topk + j];
            const __half* row = y_sorted + static_cast<size_t>(pos) * N;
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c0 + 256 * u < N) v[u] = *reinterpret_cast<const uint4*>(row + c0 + 256 * u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (c0 + 256 * u >= N) break;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float2 f;
                    if constexpr (BF) f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&v[u])[q]);
                    else f = __half22float2(reinterpret_cast<const __half2*>(&v[u])[q]);
                    acc[u][2 * q] = fmaf(wj, f.x, acc[u][2 * q]);
                    acc[u][2 * q + 1] = fmaf(wj, f.y, acc[u][2 * q + 1]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c0 + 256 * u >= N) break;
            uint4 out;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if constexpr (BF)
                    reinterpret_cast<__nv_bfloat162*>(&out)[q] = __floats2bfloat162_rn(acc[u][2 * q], acc[u][2 * q + 1]);
                else
                    reinterpret_cast<__half2*>(&out)[q] = __floats2half2_rn(acc[u][2 * q], acc[u][2 * q + 1]);
            }
            *reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * N + c0 + 256 * u) = out;
        }
    }
}

// Routed form with one expert per token, whose matmul stores each row at its
// token directly: a token whose entry took no row (an id outside [0, E)) gets
// a zero row here.  A warp per token.
__global__ void __launch_bounds__(256) moe_zero_unrouted_kernel(const int32_t* __restrict__ inv_pos, int T, int nv,
                                                                uint4* __restrict__ y)
{
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T || inv_pos[t] >= 0) return;
    uint4* row = y + static_cast<size_t>(t) * nv;
    for (int v = lane; v < nv; v += 32) row[v] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace w4a16
