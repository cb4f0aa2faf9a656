/*
 * w4a16.h -- C ABI of the B200 (sm_100a) A16W4 per-group weight-quantised
 * matmul library (libw4a16.so).
 *
 *   y[M, N] = x[M, K] . (antiquant_scale (.) W)[K, N]
 *
 * with fp16 activations x, signed int4 weights W, one fp16 scale per group
 * of g consecutive K rows and per column, and an fp16 result y (or bf16 x,
 * scale and y for W4A16_OP_DEQUANT_BF16 / w4a16_dequant_matmul_bf16).  This is the
 * operator of "WeightQuantBatchMatmulExperiment 算子深度解析"
 * (bjdmk.com.cn/news/4847346), section 4.2 (x float16/ND, weight int4/ND,
 * antiquant_scale float16/ND, y float16/ND, all 2-D).  Two algorithms compute it:
 *
 *   MSD      the multi-step decomposition of section 4.1, equations 1-11:
 *            per (row, group) A_max = max|x|; three int4 residual digits
 *            A1..A3 from 7.49*x/A_max with two x14.98 residual steps; three
 *            exact integer matmuls Y1..Y3 against the int4 weights; combined
 *            as (Y1/7.49 + Y2/(7.49*14.98) + Y3/(7.49*14.98^2))*A_max*scale
 *            and accumulated over groups (2 or 4 digits instead of 3:
 *            w4a16_msd_matmul_steps).
 *   DEQUANT  the direct dequantise-in-register W4A16 GEMM that the pages
 *            discuss as Marlin ("pwwt.cn/news/2290475", sections 1.6 and 6)
 *            and QUICK ("briefgpt.xyz/kw/cuda kernels", QUICK abstract):
 *            W' = fp16(scale * W), y = x . W' with fp32 accumulation.
 *
 * Conventions for every entry point
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    pointers marked "host" are host memory owned by the caller.  The
 *    library allocates no memory and keeps no state between calls (the one
 *    exception, w4a16_msd_matmul_noalloc, describes its own array).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  No entry point synchronises the stream, except
 *    w4a16_read_status, which says so.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed check returns an error status and launches nothing.  No entry
 *    point throws or aborts.  A failed launch returns W4A16_ERR_CUDA.
 *  - Device-side waits are bounded.  A wait that expires makes the kernel
 *    record W4A16_DEVICE_TIMEOUT in the workspace status word and return;
 *    read it with w4a16_read_status after the stream has drained.
 *  - Layouts: x row-major [M][K]; y row-major [M][N]; scale row-major
 *    [K/g][N]; logical weights as bytes [K/2][N] whose byte (i, n) holds
 *    W[2i][n] in the low nibble and W[2i+1][n] in the high nibble, two's
 *    complement ("two int4 per byte", section 4.3 of the same page).
 *  - Shape rules: M >= 0, K > 0, N > 0; N % 8 == 0; g % 32 == 0 and either
 *    128 % g == 0 (g = 32, 64, 128) or g % 128 == 0; K % g == 0.  x, y,
 *    scale and packed weights must be 16-byte aligned.  Inputs must be finite.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* w4a16_stream_t;

typedef enum {
    W4A16_OK = 0,
    W4A16_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misalignment     */
    W4A16_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. g = 96)   */
    W4A16_ERR_WORKSPACE = 3,     /* workspace missing or smaller than needed  */
    W4A16_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed      */
    W4A16_ERR_TIMEOUT = 5,       /* a device wait expired (see status word)   */
    W4A16_ERR_BAD_INDEX = 6      /* a device-side index was out of range      */
} w4a16_status;

/* Operation selector for w4a16_workspace_size, w4a16_grouped_matmul and
 * the routed (moe) entry points.  W4A16_OP_DEQUANT_BF16 is the dequant
 * variant with bf16 x, scale and y (see w4a16_dequant_matmul_bf16);
 * W4A16_OP_MSD_2STEP / _4STEP are MSD with 2 or 4 unfold steps instead of
 * 3 (see w4a16_msd_matmul_steps). */
enum {
    W4A16_OP_MSD = 0,
    W4A16_OP_DEQUANT = 1,
    W4A16_OP_DEQUANT_BF16 = 2,
    W4A16_OP_MSD_2STEP = 3,
    W4A16_OP_MSD_4STEP = 4
};

/* Bits of the device status word kept at the start of every workspace. */
enum { W4A16_DEVICE_TIMEOUT = 1u, W4A16_DEVICE_BAD_EXPERT = 2u };

/* Human-readable name of a status code (static string, never NULL). */
const char* w4a16_status_string(w4a16_status s);

/* Bytes of the packed (kernel-layout) weight buffer for a K x N int4 matrix:
 * ceil(N/128) * ceil(K/128) * 8192.  Equals K*N/2 -- the page's "two int4
 * per byte" storage (bjdmk.com.cn/news/4847346, section 4.3, the int4 weight
 * of the M=1, K=8192, N=12288 example) -- when K and N are multiples of 128;
 * the remainder of a ragged last tile or chunk is zero padding.  Returns 0
 * for non-positive sizes. */
size_t w4a16_packed_bytes(int K, int N);

/* Bytes of workspace a matmul call needs: the first stage of the page's
 * two-stage call (bjdmk.com.cn/news/4847346, section 5.4: the aclnn
 * GetWorkspaceSize query, then the execute call on a stream).
 *   op: one of the W4A16_OP_* codes; M: rows of x (for grouped calls,
 *   the total token count T); E: 1 for the dense calls, the expert count for
 *   w4a16_grouped_matmul.  The workspace holds the device status word (a
 *   256-byte header) and, for MSD, the expanded activations A_int
 *   [S][M][K] int8 and A_max [K/g][M] fp32 (the page's aUnfold workspace,
 *   section 8.2), or on decode shapes the same digits as per-piece records.
 *   Split-K partial sums never leave the chip (they meet in distributed
 *   shared memory), so the workspace holds no counters.
 * Only the status word must start at zero: zero-fill the workspace (or its
 * first 256 bytes) before its first use.  No call writes the status word
 * except to report a device error, so a workspace can be reused by later
 * calls on the same stream; after a call that reported a device error, zero
 * the status word again.  Calls that overlap in time must not share a
 * workspace.
 * Returns W4A16_ERR_INVALID_ARG / W4A16_ERR_UNSUPPORTED on bad shapes. */
w4a16_status w4a16_workspace_size(int op, int M, int K, int N, int group_size,
                                  int E, size_t* bytes);

/* a0: offline weight re-layout (the "Marlin layout" idea of pwwt.cn/news/2290475
 * section 6.2 and QUICK's offline interleave): logical packed bytes -> the
 * kernel layout, so each 128-column tile and 128-deep K chunk is one
 * contiguous 8 KB block that a single bulk copy brings into shared memory.
 *   w_logical  device, uint8 [K/2][N] (layout above)
 *   w_packed   device, w4a16_packed_bytes(K, N) bytes, written fully
 *              (padding columns/rows are written as zero weights)
 * K must be even and N % 8 == 0 (the matmul shape rules apply when the
 * packed buffer is used). */
w4a16_status w4a16_repack(const uint8_t* w_logical, int K, int N, void* w_packed,
                          w4a16_stream_t stream);

/* MSD variant, equations 1-11 of section 4.1.
 *   x          device fp16 [M][K]
 *   w_packed   device, produced by w4a16_repack for (K, N)
 *   scale      device fp16 [K/g][N]
 *   y          device fp16 [M][N], fully overwritten (round-to-nearest-even)
 *   workspace  device, >= w4a16_workspace_size(W4A16_OP_MSD, M, K, N, g, 1)
 * Step 1-8 (A_max and the residual digits, binary32 arithmetic with the
 * constants 7.49f and 14.98f) run in one kernel that writes A_int and A_max
 * to the workspace; steps 9-11 (tcgen05 int8 MMAs with exact int32
 * accumulators, the combine and the group accumulation in fp32) in a second.
 * M == 0 is a no-op. */
w4a16_status w4a16_msd_matmul(const void* x, const void* w_packed, const void* scale,
                              int M, int K, int N, int group_size, void* y,
                              void* workspace, size_t workspace_bytes,
                              w4a16_stream_t stream);

/* MSD with a chosen number of unfold steps S (2, 3 or 4): the residual
 * recursion of section 4.1 (tmp_{i+1} = (tmp_i - A_i) * 14.98f, A_{i+1} =
 * round(tmp_{i+1}), binary32) runs for S digits, and equation 10 gets one
 * term per digit, Y_i / (7.49 * 14.98^(i-1)).  Section 7 of the same page
 * notes that the speed-up varies with the number of unfold steps: fewer
 * steps do less integer work and truncate at 0.5 / (7.49 * 14.98^(S-1)) of
 * A_max * |scale| * sum|W| per group instead of 0.5 / (7.49 * 14.98^2).
 * S = 3 is w4a16_msd_matmul.  Arguments as w4a16_msd_matmul, the workspace
 * sized for W4A16_OP_MSD_2STEP / W4A16_OP_MSD / W4A16_OP_MSD_4STEP.  Any
 * other S returns W4A16_ERR_INVALID_ARG. */
w4a16_status w4a16_msd_matmul_steps(int steps, const void* x, const void* w_packed,
                                    const void* scale, int M, int K, int N, int group_size,
                                    void* y, void* workspace, size_t workspace_bytes,
                                    w4a16_stream_t stream);

/* Direct dequant variant: W' = fp16(scale * W) in registers, y = x . W' on
 * the fp16 tensor cores with fp32 accumulation, y rounded to fp16 once.
 * Arguments as w4a16_msd_matmul (workspace sized for W4A16_OP_DEQUANT). */
w4a16_status w4a16_dequant_matmul(const void* x, const void* w_packed, const void* scale,
                                  int M, int K, int N, int group_size, void* y,
                                  void* workspace, size_t workspace_bytes,
                                  w4a16_stream_t stream);

/* Direct dequant variant with bf16 activations: the INT4 weight + BF16
 * activation pairing of the Humming article (aihirek.info, supported
 * formats).  bf16 holds 8 significant bits, too few for scale * w, so the
 * weights enter the bf16 tensor cores exactly (small integers) and each
 * group's fp32 sum is multiplied by its scale in fp32:
 *   y[m][n] = bf16( sum_j scale[j][n] * sum_{k in group j} x[m][k] * W[k][n] )
 * with fp32 accumulation, y rounded to bf16 (nearest even) once.
 *   x          device bf16 [M][K]
 *   w_packed   device, produced by w4a16_repack for (K, N)
 *   scale      device bf16 [K/g][N]
 *   y          device bf16 [M][N], fully overwritten
 *   workspace  device, >= w4a16_workspace_size(W4A16_OP_DEQUANT_BF16, M, K, N, g, 1)
 * Shape and alignment rules as for the other entry points.  M == 0 is a
 * no-op. */
w4a16_status w4a16_dequant_matmul_bf16(const void* x, const void* w_packed, const void* scale,
                                       int M, int K, int N, int group_size, void* y,
                                       void* workspace, size_t workspace_bytes,
                                       w4a16_stream_t stream);

/* Grouped-expert (MoE) form: expert e multiplies the contiguous token rows
 * offsets[e] .. offsets[e+1]-1 of x by its own weights (the dense and MoE
 * scheduling Humming describes, aihirek.info "Humming ..." article).
 *   op         any W4A16_OP_* code
 *   x          device fp16 [T][K] (bf16 for W4A16_OP_DEQUANT_BF16), tokens
 *              sorted by expert
 *   w_packed   host array of E device pointers (each from w4a16_repack)
 *   scale      host array of E device pointers, fp16 [K/g][N] each (bf16
 *              for W4A16_OP_DEQUANT_BF16)
 *   offsets    device int32 [E+1], non-decreasing, offsets[0] = 0,
 *              offsets[E] = T (empty experts allowed)
 *   y          device fp16 [T][N] (bf16 for W4A16_OP_DEQUANT_BF16), fully
 *              overwritten
 *   workspace  >= w4a16_workspace_size(op, T, K, N, g, E)
 * 1 <= E <= 64.  Offsets that break the rules above give undefined rows
 * but no out-of-bounds access: rows are clamped to [0, T). */
w4a16_status w4a16_grouped_matmul(int op, const void* x, const void* const* w_packed,
                                  const void* const* scale, const int32_t* offsets,
                                  int E, int T, int K, int N, int group_size, void* y,
                                  void* workspace, size_t workspace_bytes,
                                  w4a16_stream_t stream);

/* ---- routing prep of the grouped form (mixture of experts) --------------
 * A router gives, per token t, topk expert ids topk_ids[t][j] and gate
 * weights.  The grouped matmul wants each expert's rows contiguous; the
 * steps below group the router's entries i = t*topk + j by expert, gather x
 * into that order, run the grouped matmul and add each token's rows back
 * with its gate weights -- the dense/MoE scheduling of the Humming article
 * (aihirek.info, MoE section) from the moe_align_block_size-style routing
 * step of the FlagGems operator list (pwwt.cn).  Plain reading taken: a
 * stable grouping (increasing i within an expert); an id outside [0, E)
 * takes no row, contributes nothing and sets W4A16_DEVICE_BAD_EXPERT. */

/* Stable grouping of the entries by expert.
 *   topk_ids      device int32 [T][topk]
 *   offsets       device int32 [E+1]: offsets[e] = entries whose expert < e
 *   sorted_token  device int32 [T*topk]: row r of the sorted order holds
 *                 the token of its entry; rows >= offsets[E] hold -1
 *   inv_pos       device int32 [T*topk]: the row of entry i, or -1
 *   workspace     device, >= 256 bytes, status word at its start (zeroed
 *                 by the caller before first use)
 * 1 <= E <= 64, topk >= 1, T >= 0, T*topk < 2^31. */
w4a16_status w4a16_moe_align(const int32_t* topk_ids, int T, int topk, int E, int32_t* offsets,
                             int32_t* sorted_token, int32_t* inv_pos, void* workspace,
                             size_t workspace_bytes, w4a16_stream_t stream);

/* x_sorted[r] = x[sorted_token[r]] (rows of K 16-bit values, fp16 or bf16:
 * copied as bits; zero where sorted_token[r] < 0).  x, x_sorted 16-byte
 * aligned, K % 8 == 0. */
w4a16_status w4a16_moe_gather(const void* x, const int32_t* sorted_token, int rows, int K,
                              void* x_sorted, w4a16_stream_t stream);

/* y[t] = sum_j topk_weights[t][j] * y_sorted[inv_pos[t*topk+j]] (fp16 rows of
 * N values, fp32 sums in increasing j, entries with inv_pos < 0 skipped,
 * fp16 out).  y_sorted, y 16-byte aligned, N % 8 == 0. */
w4a16_status w4a16_moe_combine(const void* y_sorted, const int32_t* inv_pos,
                               const float* topk_weights, int T, int topk, int N, void* y,
                               w4a16_stream_t stream);

/* w4a16_moe_combine on bf16 rows (bf16 in, fp32 sums, bf16 out). */
w4a16_status w4a16_moe_combine_bf16(const void* y_sorted, const int32_t* inv_pos,
                                    const float* topk_weights, int T, int topk, int N, void* y,
                                    w4a16_stream_t stream);

/* Workspace of w4a16_moe_matmul: the grouped matmul's own workspace for
 * T*topk rows, then offsets, sorted_token, inv_pos, the gathered x and the
 * per-row y. */
w4a16_status w4a16_moe_workspace_size(int op, int T, int topk, int K, int N, int group_size,
                                      int E, size_t* bytes);

/* The routed grouped form end to end: align, gather, grouped matmul,
 * combine, on one stream, no host synchronisation.  With topk == 1 the
 * combine is fused into the grouped matmul's stores (each row written at its
 * token times the gate weight; a token whose id lies outside [0, E) gets a
 * zero row).  x fp16 [T][K], y fp16
 * [T][N] (both bf16 for W4A16_OP_DEQUANT_BF16); w_packed / scale as
 * w4a16_grouped_matmul; topk_ids, topk_weights device [T][topk]. */
w4a16_status w4a16_moe_matmul(int op, const void* x, const int32_t* topk_ids,
                              const float* topk_weights, const void* const* w_packed,
                              const void* const* scale, int E, int T, int topk, int K, int N,
                              int group_size, void* y, void* workspace, size_t workspace_bytes,
                              w4a16_stream_t stream);

/* Debug window into MSD equation 9: the exact int32 Y1, Y2, Y3 per group
 * for rows m0..m1-1 and columns n0..n1-1, as accumulated by the tensor
 * cores, plus A_max.
 *   yint  device int32 [3][m1-m0][K/g][n1-n0]
 *   amax  device fp32 [m1-m0][K/g]
 *   workspace as for w4a16_msd_matmul.
 * 0 <= m0 < m1 <= M, 0 <= n0 < n1 <= N.  The full tensor is 12*M*N*K/g
 * bytes, so keep windows small. */
w4a16_status w4a16_msd_debug_yint(const void* x, const void* w_packed, int M, int K,
                                  int N, int group_size, int m0, int m1, int n0, int n1,
                                  int32_t* yint, float* amax, void* workspace,
                                  size_t workspace_bytes, w4a16_stream_t stream);

/* The same window for S = 2, 3 or 4 unfold steps (w4a16_msd_matmul_steps):
 * yint device int32 [S][m1-m0][K/g][n1-n0]; workspace sized for the op of S. */
w4a16_status w4a16_msd_debug_yint_steps(int steps, const void* x, const void* w_packed,
                                        int M, int K, int N, int group_size, int m0, int m1,
                                        int n0, int n1, int32_t* yint, float* amax,
                                        void* workspace, size_t workspace_bytes,
                                        w4a16_stream_t stream);

/* MSD matmul for callers that cannot allocate device memory.
 * No counterpart in the paper: this entry point exists for callers that have
 * no way to obtain scratch memory -- for instance a plug-in running inside a
 * host program whose memory pool owns the whole device, or a latency-critical
 * path where cudaMalloc's implicit device synchronisation is not acceptable.
 * It computes exactly what w4a16_msd_matmul computes (same kernels, same
 * arguments minus the workspace) but keeps its scratch (the status word and
 * the expanded activations: A_int and A_max, or the decode kernels' digit
 * records) in one array of W4A16_NOALLOC_SCRATCH_BYTES bytes that the
 * library declares in device memory; every GPU that loads the library holds
 * that array until the process exits.  It allocates nothing and calls no
 * allocating routine.
 *  - Calls whose scratch would exceed the array (see w4a16_workspace_size
 *    with W4A16_OP_MSD and E = 1) return W4A16_ERR_WORKSPACE and launch nothing.
 *  - The first call on a device (in a given CUDA context) looks up the
 *    array's device address (cudaGetSymbolAddress) with that device current
 *    and keeps it for later calls in the same context; make that first call
 *    before any stream capture.  A call made in a context other than the one
 *    the address was looked up in (for instance after cudaDeviceReset) looks
 *    it up again, so it too must come before any capture.
 *  - All calls share the one array and it keeps the previous call's
 *    contents.  Only the status word must start at zero; each call zeroes it
 *    on `stream` before its kernels run.  Calls that may overlap on the GPU
 *    (different streams, or different host threads) race on the array:
 *    serialise them.
 *  - A device-side wait timeout is recorded only in the array's status word,
 *    which this entry point does not report. */
#define W4A16_NOALLOC_SCRATCH_BYTES (8u << 20)
w4a16_status w4a16_msd_matmul_noalloc(const void* x, const void* w_packed, const void* scale,
                                      int M, int K, int N, int group_size, void* y,
                                      w4a16_stream_t stream);

/* Copy the device status word at the start of `workspace` into *status
 * (0 = no device error; W4A16_DEVICE_TIMEOUT bit = a bounded wait expired;
 * W4A16_DEVICE_BAD_EXPERT bit = a router id outside [0, E)).
 * SYNCHRONISES `stream`.  Returns W4A16_ERR_TIMEOUT when the timeout bit is
 * set, else W4A16_ERR_BAD_INDEX when the bad-expert bit is set, else
 * W4A16_OK. */
w4a16_status w4a16_read_status(const void* workspace, w4a16_stream_t stream,
                               uint32_t* status);

/* Set the bound on every device-side wait, in nanoseconds of GPU global
 * time (default 2e9).  Applies to launches made after the call, process-wide. */
void w4a16_set_wait_timeout_ns(uint64_t ns);

/* Launch a self-test kernel whose single wait is on a barrier that nothing
 * completes, bounded by `timeout_ns`; it must record W4A16_DEVICE_TIMEOUT in
 * the workspace status word and return.  Used to test the timeout path
 * without hanging a GPU.  workspace: device, >= 256 bytes. */
w4a16_status w4a16_selftest_wait_timeout(void* workspace, uint64_t timeout_ns,
                                         w4a16_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
