/*
 * sgq.h -- C ABI of libsgq: activation-sparse GEMV over group-wise int4 weights
 * for NVIDIA B200 (sm_100a).
 *
 * The operation ("Enabling Dynamic Sparsity in Quantized LLM Inference",
 * Abstract): weights are quantized group-wise to low-bit codes, the input
 * activation of a decode step is dynamically sparse, the active channel
 * indices are gathered at run time, and a GEMV reads only the weights of the
 * active channels:
 *
 *     y[b][n] = sum over k in S of  s[g(k)][n] * (q[k][n] - z[g(k)][n]) * x[b][k]
 *     S       = { k : |x[b][k]| > t[b] for some row b }          (strict)
 *
 * With t = 0, S is the set of nonzero channels, which is how a ReGLU FFN skips
 * its zero neurons ("SVD Contextual Sparsity Predictors for Fast LLM
 * Inference", Abstract).
 *
 * Conventions for every call:
 *  - Pointers named *_host are host memory; every other pointer is device
 *    memory owned by the caller (the library allocates nothing, frees nothing
 *    and never synchronises the stream or the device).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream); all work
 *    is enqueued asynchronously on it, in call order.
 *  - Element types: fp16 and bf16 are passed as 16-bit IEEE / bfloat16 bit
 *    patterns; all arrays are dense and row-major as stated.
 *  - Device pointers must be 16-byte aligned.
 *  - Return value: SGQ_OK (0) or a negative SGQ_ERR_* code. Argument errors are
 *    detected on the host before anything is enqueued. SGQ_ERR_CUDA means a
 *    launch failed; sgq_last_cuda_error() returns the cudaError_t.
 *  - Faults found on the device (non-finite weights, indices out of range) are
 *    OR-ed as SGQ_STATUS_* bits into an optional caller-owned int32 `status`
 *    word in device memory (NULL = not reported). The offending work is
 *    skipped, never performed out of bounds.
 *  - Only one GPU is used: the current device of the calling thread.
 */
#ifndef SGQ_H
#define SGQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SGQ_LAYOUT_VERSION 1
#define SGQ_MAX_BATCH 16

/* Return codes. */
#define SGQ_OK              0
#define SGQ_ERR_NULL       -1  /* a required pointer is NULL                     */
#define SGQ_ERR_SHAPE      -2  /* N, K, B or a size out of range / indivisible   */
#define SGQ_ERR_GROUP      -3  /* group size not 32, 64 or 128                   */
#define SGQ_ERR_ALIGN      -4  /* a device pointer is not 16-byte aligned        */
#define SGQ_ERR_BATCH      -5  /* B < 1 or B > SGQ_MAX_BATCH                     */
#define SGQ_ERR_WORKSPACE  -6  /* workspace smaller than sgq_gemv_workspace_bytes */
#define SGQ_ERR_ACT        -7  /* unknown activation                             */
#define SGQ_ERR_CUDA       -8  /* a CUDA runtime call or launch failed           */
#define SGQ_ERR_DEVICE     -9  /* current device is not compute capability 10.x  */
#define SGQ_ERR_TOO_LARGE -10  /* N above SGQ_NOALLOC_MAX_N (no-allocation entry)  */

/* Device status bits (OR-ed into the optional `status` word). */
#define SGQ_STATUS_NONFINITE_W  1  /* sgq_pack: W holds NaN or Inf (that group packed as zeros) */
#define SGQ_STATUS_BAD_INDEX    2  /* sgq_gemv: an index outside [0, K) was skipped             */
#define SGQ_STATUS_BAD_COUNT    4  /* sgq_gemv: *count outside [0, K]; clamped                  */
#define SGQ_STATUS_TIMEOUT      8  /* a bounded wait inside a GEMV kernel ran out: y is not valid */
/* After SGQ_STATUS_TIMEOUT the tensor-core kernel may have freed its tensor
 * memory with MMAs still in flight: treat it as fatal for the results of that
 * context until the stream has drained. */

/* Activations for sgq_glu. */
#define SGQ_ACT_SILU 0
#define SGQ_ACT_RELU 1

/*
 * Sizes of the packed buffers for an N x K weight with the given group size.
 *   qweight_bytes = K * N / 2          (uint8, layout below)
 *   sz_bytes      = (K / group) * N * 4 (two fp16 per group and output)
 * Requires N % 32 == 0, K % group == 0, group in {32, 64, 128}.
 */
int sgq_packed_sizes(int N, int K, int group, size_t *qweight_bytes, size_t *sz_bytes);

/*
 * Group-wise asymmetric int4 quantization of W and packing into the
 * channel-major layout, version 1 (the abstract's group-wise quantization; the
 * layout is this library's own: it keeps each input channel's codes
 * contiguous so that skipping a channel skips one contiguous run of bytes).
 *
 *   W       fp16 [N][K] (torch.nn.Linear weight layout), read only.
 *   qweight uint8 [K][N/2]: byte b of row k = q[2b][k] | q[2b+1][k] << 4.
 *   sz      [K/group][N] pairs of fp16 (scale, zero), scale first.
 * Per output n and group of `group` consecutive k: lo = min(0, min w),
 * hi = max(0, max w), s = fp16(RN((hi - lo) / 15)), z = clamp(rint(-lo/s), 0, 15),
 * q = clamp(rint(w / s) + z, 0, 15) in fp64 arithmetic, rint = half to even;
 * a group with s == 0 gets s = 1, z = 0. A group holding NaN/Inf is packed as
 * s = 1, z = 0, q = 0 and sets SGQ_STATUS_NONFINITE_W.
 * Offline step; not tuned for speed.
 */
int sgq_pack(const void *W, int N, int K, int group, void *qweight, void *sz,
             int32_t *status, void *stream);

/*
 * Runtime gathering of the active channels (the abstract's "compact runtime
 * mechanism that gathers sparse indices").
 *
 *   x       bf16 [B][K]; t_host: B floats (host memory, read during the call).
 *   idx     int32 [K] capacity; receives the ascending, unique active channels
 *           k with |x[b][k]| > t[b] for at least one b (NaN never active).
 *   count   int32 device scalar; receives |S|.
 * Requires 1 <= B <= 16, K % 8 == 0. t < 0 selects every channel.
 */
int sgq_select(const void *x, int B, int K, const float *t_host,
               int32_t *idx, int32_t *count, void *stream);

/*
 * The same active set as a bitmask, one bit per channel: the compact form an
 * activation predictor or a previous kernel can emit instead of an index list
 * (the bitmask indexing of "SparseDecoding: Decoding-Aware Pruning for
 * Accurate and Efficient LLM Inference", Abstract; the shared-memory bitmap
 * decoding of "Unified Static-Dynamic Pruning for Efficient LLM Inference",
 * Abstract, listed on that page).
 *
 *   mask    uint32 [(K + 31) / 32]: bit k % 32 of word k / 32 is 1 when
 *           |x[b][k]| > t[b] for some b (strict; NaN never active). Bits of
 *           channels k >= K in the last word are written 0.
 *   count   optional int32 device scalar (NULL = not written): |S|.
 * Requires 1 <= B <= 16, K % 8 == 0. K/8 bytes instead of 4|S| bytes.
 */
int sgq_select_mask(const void *x, int B, int K, const float *t_host,
                    uint32_t *mask, int32_t *count, void *stream);

/*
 * Workspace for sgq_gemv / sgq_gemv_thresh / sgq_gemv_dense: B*N floats of
 * split-K partial sums. It must be zero-filled once when it is allocated;
 * every call leaves it zero-filled again. Calls that may run concurrently
 * (different streams) must not share a workspace.
 *
 * Each GEMV call enqueues two kernels with programmatic dependent launch: the
 * GEMV (which reads the packed weights before the previous kernel in the
 * stream has finished, and x, idx, count only after) and a small epilogue that
 * writes y. Do not write the packed weights in the kernel that immediately
 * precedes a GEMV call in the same stream without a full stream dependency.
 */
size_t sgq_gemv_workspace_bytes(int N, int K, int B);

/*
 * The activation-sparse GEMV: y[b][n] = sum over i < *count of
 * s (q - z) of (n, idx[i]) times x[b][idx[i]] (bf16 output, round to nearest
 * even; fp32 accumulation). Every batch row uses the same active list
 * (normally the union from sgq_select); rows are not masked inside it.
 *
 *   qweight, sz  packed by sgq_pack (layout version 1) for this N, K, group.
 *   x            bf16 [B][K].
 *   idx, count   device list and device count (as written by sgq_select).
 *                Indices should ascend (any order in [0, K) is correct, only
 *                slower); an index outside [0, K) is skipped and flagged.
 *   y            bf16 [B][N] output.
 *   y_f32        optional fp32 [B][N] copy of y before the bf16 rounding
 *                (NULL = not written).
 *   workspace    see sgq_gemv_workspace_bytes.
 * The grid is fixed by (N, K, B, SM count), not by *count: nothing is read
 * back to the host.
 */
int sgq_gemv(const void *qweight, const void *sz, int N, int K, int group,
             const void *x, int B, const int32_t *idx, const int32_t *count,
             void *y, float *y_f32, void *workspace, size_t ws_bytes,
             int32_t *status, void *stream);

/*
 * Threshold and GEMV in one launch: the same result as sgq_select(x, t) followed
 * by sgq_gemv on its output, with the selection done by each CTA for its own
 * slice of channels (no index list in memory). B == 1 only.
 */
int sgq_gemv_thresh(const void *qweight, const void *sz, int N, int K, int group,
                    const void *x, float t, void *y, float *y_f32,
                    void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * The same at batch B (1..16) with one threshold per batch row: the result of
 * sgq_select(x, B, t_host) (the union of the rows' active channels, "Enabling
 * Dynamic Sparsity in Quantized LLM Inference", Abstract: runtime gathering of
 * the active indices) followed by sgq_gemv over that list, in one GEMV launch
 * (plus the epilogue kernel): each CTA thresholds all B rows of its own slice
 * of channels, so no index list is written or read.
 *
 *   x        bf16 [B][K], K a multiple of 8.
 *   t_host   host array of B floats; channel k is active when |x[b][k]| > t[b]
 *            for some b (strict; NaN never; t < 0 selects every channel).
 *   y, y_f32, workspace, status, stream  as sgq_gemv (workspace for B rows).
 * Returns as sgq_gemv; SGQ_ERR_BATCH for B outside 1..16, SGQ_ERR_NULL for a
 * NULL t_host.
 */
int sgq_gemv_thresh_batch(const void *qweight, const void *sz, int N, int K, int group,
                          const void *x, int B, const float *t_host, void *y, float *y_f32,
                          void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * Accumulating forms: y_acc += W_deq[:, S] x[S] into a caller-owned fp32
 * buffer y_acc [B][N] (16-byte aligned), e.g. the fp32 residual stream of a
 * decode step (the pages fuse no such epilogue; it is a deployment form of
 * this library). The GEMV's split-K partial sums are added straight into
 * y_acc with fp32 reductions, so there is no workspace, no bf16 rounding and
 * no second (epilogue) kernel: one launch per call. The order of the fp32
 * additions is not fixed, so the low bits of y_acc may differ from run to
 * run. Rows as sgq_gemv (index list, B <= 16) or sgq_gemv_thresh (B = 1).
 */
int sgq_gemv_acc(const void *qweight, const void *sz, int N, int K, int group,
                 const void *x, int B, const int32_t *idx, const int32_t *count,
                 float *y_acc, int32_t *status, void *stream);
int sgq_gemv_thresh_acc(const void *qweight, const void *sz, int N, int K, int group,
                        const void *x, float t, float *y_acc, int32_t *status, void *stream);

/*
 * The activation-sparse GEMV with the active set given as a bitmask (as
 * written by sgq_select_mask, or by any producer of the same format): the
 * same result as sgq_gemv over the ascending list of the set bits. Each CTA
 * decodes the bits of its own channel slice in shared memory, so no global
 * list or count is needed. Bits of channels >= K are ignored. 1 <= B <= 16;
 * every batch row uses the one mask (normally the union). Other arguments as
 * sgq_gemv.
 */
int sgq_gemv_mask(const void *qweight, const void *sz, int N, int K, int group,
                  const void *x, int B, const uint32_t *mask, void *y, float *y_f32,
                  void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * The dense int4 GEMV over the same packed weights (every channel active): the
 * dense quantized inference that the abstract compares against.
 */
int sgq_gemv_dense(const void *qweight, const void *sz, int N, int K, int group,
                   const void *x, int B, void *y, float *y_f32,
                   void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * Static 2:4 weight sparsity composed with the dynamic activation sparsity
 * (the N:M sparse GEMV with bitmask indexing of "SparseDecoding: Decoding-
 * Aware Pruning for Accurate and Efficient LLM Inference", Abstract, placed
 * so that skipped input channels stay whole skipped runs).
 *
 * The 2:4 pattern runs along the outputs of each channel row: in every block
 * of 4 consecutive outputs, 2 are kept, and the g channels of a quantization
 * group share that choice. sgq_pack_nm prunes and packs W: per (group, block)
 * it keeps the 2 outputs with the largest sum over the group of w^2 (exact in
 * fp64; ties keep the lower output), then quantizes the kept outputs exactly
 * as sgq_pack does. Layout (N % 64 == 0):
 *   qweight u8 [K][N/4]: byte j of row k = code of slot 2j | slot 2j+1 << 4,
 *                        slots 2j, 2j+1 = the kept outputs of block j, ascending.
 *   keep    u8 [K/group][N/8]: byte j = keep nibble of block 2j | that of
 *                        block 2j+1 << 4 (bit i set = output 4 block + i kept).
 *   sz      [K/group][N/2] (fp16 scale, fp16 zero) per slot.
 * An active channel costs N/4 bytes instead of N/2. A block holding NaN/Inf
 * keeps outputs 0 and 1 as zeros and sets SGQ_STATUS_NONFINITE_W.
 *
 * sgq_gemv_nm / sgq_gemv_nm_thresh: y = W_pruned[:, S] x[S] (pruned weights
 * are zero), batch 1, rows from an index list (as sgq_gemv) or the fused
 * threshold (as sgq_gemv_thresh). Workspace as sgq_gemv with B = 1.
 */
int sgq_packed_sizes_nm(int N, int K, int group, size_t *qweight_bytes, size_t *keep_bytes,
                        size_t *sz_bytes);
int sgq_pack_nm(const void *W, int N, int K, int group, void *qweight, void *keep, void *sz,
                int32_t *status, void *stream);
int sgq_gemv_nm(const void *qweight, const void *keep, const void *sz, int N, int K, int group,
                const void *x, const int32_t *idx, const int32_t *count, void *y, float *y_f32,
                void *workspace, size_t ws_bytes, int32_t *status, void *stream);
int sgq_gemv_nm_thresh(const void *qweight, const void *keep, const void *sz, int N, int K,
                       int group, const void *x, float t, void *y, float *y_f32,
                       void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * Gated FFN activation h = act(gate) * up, elementwise over [B][I] bf16
 * (fp32 arithmetic, bf16 round-to-nearest-even output). act = SGQ_ACT_SILU
 * (v / (1 + e^-v)) or SGQ_ACT_RELU (v if v > 0 else 0, the ReGLU of the SVD
 * predictor page, whose zeros sgq_select with t = 0 then skips).
 * Requires (B * I) % 8 == 0.
 */
int sgq_glu(const void *gate, const void *up, void *h, int B, int I, int act, void *stream);

/*
 * Fused gated FFN front half: the gate and up projections of one FFN as a
 * single activation-sparse GEMV, with the activation in its epilogue:
 *
 *     h[b][i] = act(gate[b][i]) * up[b][i],   i < I,
 *     gate = W_g[:, S] x[S],  up = W_u[:, S] x[S]   (one active set S),
 *
 * where gate and up are the fp32 sums (never rounded to bf16 in between) and h
 * is rounded once to bf16 (round to nearest even); act as in sgq_glu. The
 * pages fuse nothing of the kind; the point is the decode FFN, where the gate
 * and up GEMVs read the same sparse input ("Enabling Dynamic Sparsity in
 * Quantized LLM Inference", Abstract) and ReLU gating then produces the zeros
 * that the down projection skips ("SVD Contextual Sparsity Predictors for Fast
 * LLM Inference", Abstract): the down projection is sgq_gemv_thresh on h with
 * t = 0, which finds the active channels of h in its own prologue.
 *
 *   qweight, sz  sgq_pack of the stacked weight [W_g; W_u], fp16 [2I][K]
 *                (rows 0..I-1 the gate, I..2I-1 the up projection), packed
 *                with N = 2I: each active channel is then one contiguous run
 *                of I bytes covering both projections.
 *   I            intermediate size; 2I must be a multiple of 32.
 *   h            bf16 [B][I]. h_f32: optional fp32 [B][I] copy of h before the
 *                bf16 rounding (NULL = not written).
 *   workspace    sgq_gemv_workspace_bytes(2 * I, K, B) bytes, as for sgq_gemv.
 * The three forms take the rows as sgq_gemv (index list), sgq_gemv_thresh
 * (B == 1, select fused) and sgq_gemv_dense (every channel). Returns as
 * sgq_gemv, plus SGQ_ERR_ACT for an unknown act.
 */
int sgq_gemv_glu(const void *qweight, const void *sz, int I, int K, int group,
                 const void *x, int B, const int32_t *idx, const int32_t *count, int act,
                 void *h, float *h_f32, void *workspace, size_t ws_bytes, int32_t *status,
                 void *stream);
int sgq_gemv_glu_thresh(const void *qweight, const void *sz, int I, int K, int group,
                        const void *x, float t, int act, void *h, float *h_f32,
                        void *workspace, size_t ws_bytes, int32_t *status, void *stream);
/* The fused-select form at batch B with one threshold per row (rows as
 * sgq_gemv_thresh_batch: the union of the rows' active channels). */
int sgq_gemv_glu_thresh_batch(const void *qweight, const void *sz, int I, int K, int group,
                              const void *x, int B, const float *t_host, int act, void *h,
                              float *h_f32, void *workspace, size_t ws_bytes,
                              int32_t *status, void *stream);
int sgq_gemv_glu_dense(const void *qweight, const void *sz, int I, int K, int group,
                       const void *x, int B, int act, void *h, float *h_f32,
                       void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/*
 * The whole decode FFN at batch 1, three kernels:
 *
 *     h = bf16(act(W_g[:, S] x[S]) * (W_u[:, S] x[S])),  S = { k : |x_k| > t_in }
 *     y = W_d[:, T] h[T],                                  T = { i : |h_i| > t_h }
 *
 * The gate/up GEMV (select fused) leaves its fp32 sums in the workspace; the
 * down GEMV's prologue forms h from them for its own slice of the I channels
 * (the same bf16 h as sgq_gemv_glu_thresh), selects T there and gathers only
 * those rows ("SVD Contextual Sparsity Predictors for Fast LLM Inference",
 * Abstract: with ReLU gating and t_h = 0, T is the nonzero neurons); h is not
 * written to memory unless h_out is given. The epilogue kernel writes y and
 * re-zeroes the workspace.
 *
 *   qweight_gu, sz_gu  sgq_pack of the stacked [W_g; W_u] (N = 2I, K = H).
 *   qweight_d, sz_d    sgq_pack of W_d (N = H, K = I).
 *   x                  bf16 [1][H]; y bf16 [1][H]; y_f32 optional fp32 [1][H].
 *   h_out              optional bf16 [1][I] copy of h (NULL = not written).
 *   workspace          sgq_ffn_workspace_bytes(H, I) bytes, zero-filled once.
 * Requires H % 8 == 0 and I % 8 == 0 besides the sgq_pack conditions.
 * Returns as sgq_gemv, plus SGQ_ERR_ACT.
 */
size_t sgq_ffn_workspace_bytes(int H, int I);
int sgq_ffn(const void *qweight_gu, const void *sz_gu, const void *qweight_d, const void *sz_d,
            int H, int I, int group, const void *x, float t_in, int act, float t_h, void *y,
            float *y_f32, void *h_out, void *workspace, size_t ws_bytes, int32_t *status,
            void *stream);

/*
 * sgq_gemv_thresh without a workspace argument, for callers that cannot
 * allocate device memory (no cudaMalloc available to them, or none allowed
 * during the call). The pages have no counterpart of this entry point; it is a
 * deployment convenience of this library.
 *
 * The split-K scratch is a fixed array of SGQ_NOALLOC_MAX_N floats compiled
 * into the library (held on every GPU that loads it until the process exits).
 * N > SGQ_NOALLOC_MAX_N returns SGQ_ERR_TOO_LARGE. The first call on a device
 * (that device current) looks up the array's device address once
 * (cudaGetSymbolAddress, thread-safe) and caches it, so make that first call
 * before any stream capture; the cached address is not valid across a
 * cudaDeviceReset. Every call clears the N floats it uses with
 * cudaMemsetAsync on `stream` before the GEMV, so it never depends on what an
 * earlier call left there; calls that overlap on the GPU share the array and
 * race. Nothing is allocated or freed. Other arguments as sgq_gemv_thresh.
 */
#define SGQ_NOALLOC_MAX_N 65536
int sgq_gemv_thresh_noalloc(const void *qweight, const void *sz, int N, int K, int group,
                            const void *x, float t, void *y, float *y_f32, int32_t *status,
                            void *stream);

/*
 * Read the device status word (the SGQ_STATUS_* bits that calls OR into it):
 * enqueues on `stream` a copy of *dev_status into *host_out (host memory;
 * the value is there once the stream has reached this point, e.g. after the
 * caller synchronises it), then, if `clear` is nonzero, sets *dev_status to 0.
 * Does not synchronise.
 */
int sgq_read_status(int32_t *dev_status, int32_t *host_out, int clear, void *stream);

/* Text for a return code (static string). */
const char *sgq_status_string(int code);

/* cudaError_t of the last SGQ_ERR_CUDA on this thread (0 if none). */
int sgq_last_cuda_error(void);

/* SGQ_LAYOUT_VERSION of the packed format this build reads and writes. */
int sgq_layout_version(void);

/*
 * Test hook for the device-side wait limits (not for production use):
 * sgq_gemv with B = 9..16 (the tensor-core kernel) in which the MMA issuer
 * withholds the commit that releases the last group run's accumulators. The
 * CTAs' waits on it give up after 0.2 s, SGQ_STATUS_TIMEOUT is set in *status
 * (status must be non-NULL to see it) and y is not valid; the commit that
 * covers every MMA is not withheld, so the kernel still frees its tensor
 * memory after its MMAs have completed and the context stays usable.
 * Arguments as sgq_gemv; B outside 9..16 returns SGQ_ERR_SHAPE.
 */
int sgq_debug_gemv_withhold(const void *qweight, const void *sz, int N, int K, int group,
                            const void *x, int B, const int32_t *idx, const int32_t *count,
                            void *y, float *y_f32, void *workspace, size_t ws_bytes,
                            int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SGQ_H */
