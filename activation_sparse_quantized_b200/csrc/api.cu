// api.cu -- the extern "C" entry points of libsgq (declared in include/sgq.h).
// Host-side argument checks, then one launch on the caller's stream. Nothing
// here allocates, frees or synchronises.
#include "sgq_launch.h"

#include <cuda_runtime.h>

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices];      // 0 = not queried yet
int g_device_ok[kMaxDevices];    // 0 = unknown, 1 = sm_10x, -1 = other

int fail_cuda(cudaError_t e)
{
    g_last_cuda_error = (int)e;
    return SGQ_ERR_CUDA;
}

// SM count of the current device (cached), or a negative SGQ_ERR_*.
int current_device_sms()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail_cuda(e);
    if (dev < 0 || dev >= kMaxDevices)
        return SGQ_ERR_DEVICE;
    if (g_device_ok[dev] == 0) {
        int major = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) !=
            cudaSuccess)
            return fail_cuda(e);
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) !=
            cudaSuccess)
            return fail_cuda(e);
        g_num_sms[dev] = sms;
        g_device_ok[dev] = (major == 10) ? 1 : -1;
    }
    if (g_device_ok[dev] != 1)
        return SGQ_ERR_DEVICE;
    return g_num_sms[dev];
}

bool aligned16(const void *p)
{
    return ((uintptr_t)p & 15u) == 0;
}

bool group_ok(int group)
{
    return group == 32 || group == 64 || group == 128;
}

int check_weights(int N, int K, int group)
{
    if (!group_ok(group))
        return SGQ_ERR_GROUP;
    if (N <= 0 || K <= 0 || N % 32 != 0 || K % group != 0)
        return SGQ_ERR_SHAPE;
    if ((long long)N * K > (1LL << 40))
        return SGQ_ERR_SHAPE;
    return SGQ_OK;
}

int run_gemv(sgq::GemvProblem &p, size_t ws_bytes, void *workspace, void *stream)
{
    int rc = check_weights(p.N, p.K, p.group);
    if (rc)
        return rc;
    if (p.B < 1 || p.B > SGQ_MAX_BATCH)
        return SGQ_ERR_BATCH;
    if (!p.qweight || !p.sz || !p.x || !p.y || !workspace)
        return SGQ_ERR_NULL;
    if (p.source == sgq::ROWS_LIST && (!p.idx || !p.count))
        return SGQ_ERR_NULL;
    if (p.source == sgq::ROWS_MASK && !p.mask)
        return SGQ_ERR_NULL;
    if (p.source == sgq::ROWS_MASK && !aligned16(p.mask))
        return SGQ_ERR_ALIGN;
    if (!aligned16(p.qweight) || !aligned16(p.sz) || !aligned16(p.x) || !aligned16(p.y) ||
        !aligned16(workspace) || (p.y_f32 && !aligned16(p.y_f32)))
        return SGQ_ERR_ALIGN;
    if (p.source == sgq::ROWS_THRESH && (p.K % 8 != 0 || (p.keep && p.B != 1)))
        return SGQ_ERR_SHAPE;
    if (ws_bytes < sgq::gemv_workspace_bytes(p.N, p.B))
        return SGQ_ERR_WORKSPACE;
    const int sms = current_device_sms();
    if (sms < 0)
        return sms;
    p.ws_acc = static_cast<float *>(workspace);
    cudaError_t e = sgq::launch_gemv(p, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return fail_cuda(e);
    return SGQ_OK;
}

} // namespace

int sgq::record_cuda_error(cudaError_t e)
{
    return fail_cuda(e);
}

extern "C" {

int sgq_layout_version(void)
{
    return SGQ_LAYOUT_VERSION;
}

int sgq_last_cuda_error(void)
{
    return g_last_cuda_error;
}

int sgq_read_status(int32_t *dev_status, int32_t *host_out, int clear, void *stream)
{
    if (!dev_status || !host_out)
        return SGQ_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(host_out, dev_status, sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return fail_cuda(e);
    if (clear) {
        e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), st);
        if (e != cudaSuccess)
            return fail_cuda(e);
    }
    return SGQ_OK;
}

const char *sgq_status_string(int code)
{
    switch (code) {
    case SGQ_OK: return "ok";
    case SGQ_ERR_NULL: return "a required pointer is NULL";
    case SGQ_ERR_SHAPE: return "shape out of range or not divisible as required";
    case SGQ_ERR_GROUP: return "group size must be 32, 64 or 128";
    case SGQ_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case SGQ_ERR_BATCH: return "batch must be between 1 and 16";
    case SGQ_ERR_WORKSPACE: return "workspace smaller than sgq_gemv_workspace_bytes";
    case SGQ_ERR_ACT: return "unknown activation";
    case SGQ_ERR_CUDA: return "a CUDA call failed (see sgq_last_cuda_error)";
    case SGQ_ERR_DEVICE: return "the current device is not compute capability 10.x (B200)";
    case SGQ_ERR_TOO_LARGE: return "N exceeds SGQ_NOALLOC_MAX_N, the fixed scratch of sgq_gemv_thresh_noalloc";
    default: return "unknown sgq status";
    }
}

int sgq_packed_sizes(int N, int K, int group, size_t *qweight_bytes, size_t *sz_bytes)
{
    int rc = check_weights(N, K, group);
    if (rc)
        return rc;
    if (!qweight_bytes || !sz_bytes)
        return SGQ_ERR_NULL;
    *qweight_bytes = (size_t)K * (N / 2);
    *sz_bytes = (size_t)(K / group) * N * 4;
    return SGQ_OK;
}

int sgq_pack(const void *W, int N, int K, int group, void *qweight, void *sz, int32_t *status,
             void *stream)
{
    int rc = check_weights(N, K, group);
    if (rc)
        return rc;
    if (!W || !qweight || !sz)
        return SGQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(sz))
        return SGQ_ERR_ALIGN;
    int sms = current_device_sms();
    if (sms < 0)
        return sms;
    cudaError_t e = sgq::launch_pack(static_cast<const uint16_t *>(W), N, K, group,
                                     static_cast<uint8_t *>(qweight),
                                     static_cast<uint32_t *>(sz), status,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

static int check_weights_nm(int N, int K, int group)
{
    int rc = check_weights(N, K, group);
    if (rc)
        return rc;
    return (N % 64 == 0) ? SGQ_OK : SGQ_ERR_SHAPE;
}

int sgq_packed_sizes_nm(int N, int K, int group, size_t *qweight_bytes, size_t *keep_bytes,
                        size_t *sz_bytes)
{
    int rc = check_weights_nm(N, K, group);
    if (rc)
        return rc;
    if (!qweight_bytes || !keep_bytes || !sz_bytes)
        return SGQ_ERR_NULL;
    *qweight_bytes = (size_t)K * (N / 4);
    *keep_bytes = (size_t)(K / group) * (N / 8);
    *sz_bytes = (size_t)(K / group) * (N / 2) * 4;
    return SGQ_OK;
}

int sgq_pack_nm(const void *W, int N, int K, int group, void *qweight, void *keep, void *sz,
                int32_t *status, void *stream)
{
    int rc = check_weights_nm(N, K, group);
    if (rc)
        return rc;
    if (!W || !qweight || !keep || !sz)
        return SGQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(keep) || !aligned16(sz))
        return SGQ_ERR_ALIGN;
    int sms = current_device_sms();
    if (sms < 0)
        return sms;
    cudaError_t e = sgq::launch_pack_nm(static_cast<const uint16_t *>(W), N, K, group,
                                        static_cast<uint8_t *>(qweight),
                                        static_cast<uint8_t *>(keep),
                                        static_cast<uint32_t *>(sz), status,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

int sgq_select(const void *x, int B, int K, const float *t_host, int32_t *idx, int32_t *count,
               void *stream)
{
    if (B < 1 || B > SGQ_MAX_BATCH)
        return SGQ_ERR_BATCH;
    if (K <= 0 || K % 8 != 0)
        return SGQ_ERR_SHAPE;
    if (!x || !t_host || !idx || !count)
        return SGQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(idx))
        return SGQ_ERR_ALIGN;
    int sms = current_device_sms();
    if (sms < 0)
        return sms;
    sgq::Thresholds th{};
    for (int b = 0; b < B; ++b)
        th.t[b] = t_host[b];
    cudaError_t e = sgq::launch_select(static_cast<const uint16_t *>(x), B, K, th, idx, count,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

int sgq_select_mask(const void *x, int B, int K, const float *t_host, uint32_t *mask,
                    int32_t *count, void *stream)
{
    if (B < 1 || B > SGQ_MAX_BATCH)
        return SGQ_ERR_BATCH;
    if (K <= 0 || K % 8 != 0)
        return SGQ_ERR_SHAPE;
    if (!x || !t_host || !mask)
        return SGQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(mask))
        return SGQ_ERR_ALIGN;
    int sms = current_device_sms();
    if (sms < 0)
        return sms;
    sgq::Thresholds th{};
    for (int b = 0; b < B; ++b)
        th.t[b] = t_host[b];
    cudaError_t e = sgq::launch_select_mask(static_cast<const uint16_t *>(x), B, K, th, mask,
                                            count, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

size_t sgq_gemv_workspace_bytes(int N, int K, int B)
{
    (void)K;
    if (N <= 0 || B < 1 || B > SGQ_MAX_BATCH)
        return 0;
    return sgq::gemv_workspace_bytes(N, B);
}

int sgq_gemv(const void *qweight, const void *sz, int N, int K, int group, const void *x, int B,
             const int32_t *idx, const int32_t *count, void *y, float *y_f32, void *workspace,
             size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.idx = idx;
    p.count = count;
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_LIST;
    return run_gemv(p, ws_bytes, workspace, stream);
}

int sgq_debug_gemv_withhold(const void *qweight, const void *sz, int N, int K, int group,
                            const void *x, int B, const int32_t *idx, const int32_t *count,
                            void *y, float *y_f32, void *workspace, size_t ws_bytes,
                            int32_t *status, void *stream)
{
    if (B <= 8 || B > SGQ_MAX_BATCH)
        return SGQ_ERR_SHAPE;
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.idx = idx;
    p.count = count;
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_LIST;
    p.debug_withhold_ready = 1;
    return run_gemv(p, ws_bytes, workspace, stream);
}

int sgq_gemv_thresh(const void *qweight, const void *sz, int N, int K, int group, const void *x,
                    float t, void *y, float *y_f32, void *workspace, size_t ws_bytes,
                    int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = 1;
    p.t = t;
    p.source = sgq::ROWS_THRESH;
    return run_gemv(p, ws_bytes, workspace, stream);
}

int sgq_gemv_thresh_batch(const void *qweight, const void *sz, int N, int K, int group,
                          const void *x, int B, const float *t_host, void *y, float *y_f32,
                          void *workspace, size_t ws_bytes, int32_t *status, void *stream)
{
    if (B < 1 || B > SGQ_MAX_BATCH)
        return SGQ_ERR_BATCH;
    if (!t_host)
        return SGQ_ERR_NULL;
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.t = t_host[0];
    for (int b = 0; b < B; ++b)
        p.tb[b] = t_host[b];
    p.source = sgq::ROWS_THRESH;
    return run_gemv(p, ws_bytes, workspace, stream);
}

// Accumulating forms: y_acc [B][N] fp32 (caller-owned) += the GEMV; the GEMV
// kernel's split-K reductions land in y_acc itself, so there is no workspace
// and no epilogue kernel.
static int run_gemv_acc(sgq::GemvProblem &p, float *y_acc, void *stream)
{
    if (!y_acc)
        return SGQ_ERR_NULL;
    p.accumulate = true;
    p.y = reinterpret_cast<uint16_t *>(y_acc); // non-null for the checks; never written
    return run_gemv(p, sgq::gemv_workspace_bytes(p.N, p.B), y_acc, stream);
}

int sgq_gemv_acc(const void *qweight, const void *sz, int N, int K, int group, const void *x,
                 int B, const int32_t *idx, const int32_t *count, float *y_acc, int32_t *status,
                 void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.idx = idx;
    p.count = count;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_LIST;
    return run_gemv_acc(p, y_acc, stream);
}

int sgq_gemv_thresh_acc(const void *qweight, const void *sz, int N, int K, int group,
                        const void *x, float t, float *y_acc, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = 1;
    p.t = t;
    p.source = sgq::ROWS_THRESH;
    return run_gemv_acc(p, y_acc, stream);
}

int sgq_gemv_mask(const void *qweight, const void *sz, int N, int K, int group, const void *x,
                  int B, const uint32_t *mask, void *y, float *y_f32, void *workspace,
                  size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.mask = mask;
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_MASK;
    return run_gemv(p, ws_bytes, workspace, stream);
}

static int run_gemv_nm(sgq::GemvProblem &p, const void *keep, size_t ws_bytes, void *workspace,
                       void *stream)
{
    int rc = check_weights_nm(p.N, p.K, p.group);
    if (rc)
        return rc;
    if (!keep)
        return SGQ_ERR_NULL;
    if (!aligned16(keep))
        return SGQ_ERR_ALIGN;
    p.keep = static_cast<const uint8_t *>(keep);
    return run_gemv(p, ws_bytes, workspace, stream);
}

int sgq_gemv_nm(const void *qweight, const void *keep, const void *sz, int N, int K, int group,
                const void *x, const int32_t *idx, const int32_t *count, void *y, float *y_f32,
                void *workspace, size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.idx = idx;
    p.count = count;
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = 1;
    p.source = sgq::ROWS_LIST;
    return run_gemv_nm(p, keep, ws_bytes, workspace, stream);
}

int sgq_gemv_nm_thresh(const void *qweight, const void *keep, const void *sz, int N, int K,
                       int group, const void *x, float t, void *y, float *y_f32, void *workspace,
                       size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = 1;
    p.t = t;
    p.source = sgq::ROWS_THRESH;
    return run_gemv_nm(p, keep, ws_bytes, workspace, stream);
}

int sgq_gemv_dense(const void *qweight, const void *sz, int N, int K, int group, const void *x,
                   int B, void *y, float *y_f32, void *workspace, size_t ws_bytes,
                   int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.y_f32 = y_f32;
    p.status = status;
    p.N = N;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_DENSE;
    return run_gemv(p, ws_bytes, workspace, stream);
}

// Fused gate + up + GLU: one GEMV over the stacked [gate; up] weights
// (N = 2I outputs) whose epilogue writes h = act(gate) * up.
static int run_gemv_glu(sgq::GemvProblem &p, int I, int act, size_t ws_bytes, void *workspace,
                        void *stream)
{
    if (act != SGQ_ACT_SILU && act != SGQ_ACT_RELU)
        return SGQ_ERR_ACT;
    if (I <= 0 || I > (1 << 29))
        return SGQ_ERR_SHAPE;
    p.N = 2 * I;
    p.epilogue = (act == SGQ_ACT_SILU) ? sgq::EPI_GLU_SILU : sgq::EPI_GLU_RELU;
    return run_gemv(p, ws_bytes, workspace, stream);
}

int sgq_gemv_glu(const void *qweight, const void *sz, int I, int K, int group, const void *x,
                 int B, const int32_t *idx, const int32_t *count, int act, void *h,
                 float *h_f32, void *workspace, size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.idx = idx;
    p.count = count;
    p.y = static_cast<uint16_t *>(h);
    p.y_f32 = h_f32;
    p.status = status;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_LIST;
    return run_gemv_glu(p, I, act, ws_bytes, workspace, stream);
}

int sgq_gemv_glu_thresh(const void *qweight, const void *sz, int I, int K, int group,
                        const void *x, float t, int act, void *h, float *h_f32, void *workspace,
                        size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(h);
    p.y_f32 = h_f32;
    p.status = status;
    p.K = K;
    p.group = group;
    p.B = 1;
    p.t = t;
    p.source = sgq::ROWS_THRESH;
    return run_gemv_glu(p, I, act, ws_bytes, workspace, stream);
}

int sgq_gemv_glu_thresh_batch(const void *qweight, const void *sz, int I, int K, int group,
                              const void *x, int B, const float *t_host, int act, void *h,
                              float *h_f32, void *workspace, size_t ws_bytes, int32_t *status,
                              void *stream)
{
    if (B < 1 || B > SGQ_MAX_BATCH)
        return SGQ_ERR_BATCH;
    if (!t_host)
        return SGQ_ERR_NULL;
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(h);
    p.y_f32 = h_f32;
    p.status = status;
    p.K = K;
    p.group = group;
    p.B = B;
    p.t = t_host[0];
    for (int b = 0; b < B; ++b)
        p.tb[b] = t_host[b];
    p.source = sgq::ROWS_THRESH;
    return run_gemv_glu(p, I, act, ws_bytes, workspace, stream);
}

int sgq_gemv_glu_dense(const void *qweight, const void *sz, int I, int K, int group,
                       const void *x, int B, int act, void *h, float *h_f32, void *workspace,
                       size_t ws_bytes, int32_t *status, void *stream)
{
    sgq::GemvProblem p{};
    p.qweight = static_cast<const uint8_t *>(qweight);
    p.sz = static_cast<const uint32_t *>(sz);
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(h);
    p.y_f32 = h_f32;
    p.status = status;
    p.K = K;
    p.group = group;
    p.B = B;
    p.source = sgq::ROWS_DENSE;
    return run_gemv_glu(p, I, act, ws_bytes, workspace, stream);
}

size_t sgq_ffn_workspace_bytes(int H, int I)
{
    if (H <= 0 || I <= 0 || I > (1 << 29))
        return 0;
    return sgq::gemv_workspace_bytes(2 * I, 1) + sgq::gemv_workspace_bytes(H, 1);
}

int sgq_ffn(const void *qweight_gu, const void *sz_gu, const void *qweight_d, const void *sz_d,
            int H, int I, int group, const void *x, float t_in, int act, float t_h, void *y,
            float *y_f32, void *h_out, void *workspace, size_t ws_bytes, int32_t *status,
            void *stream)
{
    if (act != SGQ_ACT_SILU && act != SGQ_ACT_RELU)
        return SGQ_ERR_ACT;
    if (I <= 0 || I > (1 << 29) || H <= 0)
        return SGQ_ERR_SHAPE;
    int rc = check_weights(2 * I, H, group);
    if (rc)
        return rc;
    rc = check_weights(H, I, group);
    if (rc)
        return rc;
    if (H % 8 != 0 || I % 8 != 0)
        return SGQ_ERR_SHAPE;
    if (!qweight_gu || !sz_gu || !qweight_d || !sz_d || !x || !y || !workspace)
        return SGQ_ERR_NULL;
    if (!aligned16(qweight_gu) || !aligned16(sz_gu) || !aligned16(qweight_d) ||
        !aligned16(sz_d) || !aligned16(x) || !aligned16(y) || !aligned16(workspace) ||
        (y_f32 && !aligned16(y_f32)) || (h_out && !aligned16(h_out)))
        return SGQ_ERR_ALIGN;
    if (ws_bytes < sgq_ffn_workspace_bytes(H, I))
        return SGQ_ERR_WORKSPACE;
    const int sms = current_device_sms();
    if (sms < 0)
        return sms;
    float *gu = static_cast<float *>(workspace);
    float *wsd = gu + sgq::gemv_workspace_bytes(2 * I, 1) / sizeof(float);
    // gate and up as one accumulating GEMV (select fused): fp32 sums into gu
    sgq::GemvProblem p1{};
    p1.qweight = static_cast<const uint8_t *>(qweight_gu);
    p1.sz = static_cast<const uint32_t *>(sz_gu);
    p1.x = static_cast<const uint16_t *>(x);
    p1.status = status;
    p1.N = 2 * I;
    p1.K = H;
    p1.group = group;
    p1.B = 1;
    p1.t = t_in;
    p1.source = sgq::ROWS_THRESH;
    p1.accumulate = true;
    p1.ws_acc = gu;
    cudaError_t e = sgq::launch_gemv(p1, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return fail_cuda(e);
    // the down projection: h = bf16(act(gate) * up) and its active channels
    // in the prologue, then the GEMV and the epilogue kernel (which re-zeroes gu)
    sgq::GemvProblem p2{};
    p2.qweight = static_cast<const uint8_t *>(qweight_d);
    p2.sz = static_cast<const uint32_t *>(sz_d);
    p2.x = static_cast<const uint16_t *>(x); // not read (rows come from gu)
    p2.y = static_cast<uint16_t *>(y);
    p2.y_f32 = y_f32;
    p2.status = status;
    p2.N = H;
    p2.K = I;
    p2.group = group;
    p2.B = 1;
    p2.t = t_h;
    p2.source = sgq::ROWS_GLU;
    p2.gu = gu;
    p2.glu_act = act;
    p2.h_out = static_cast<uint16_t *>(h_out);
    p2.zero_extra = gu;
    p2.zero_extra_n = 2 * I;
    p2.ws_acc = wsd;
    e = sgq::launch_gemv(p2, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

int sgq_glu(const void *gate, const void *up, void *h, int B, int I, int act, void *stream)
{
    if (act != SGQ_ACT_SILU && act != SGQ_ACT_RELU)
        return SGQ_ERR_ACT;
    if (B < 1 || I <= 0 || ((long long)B * I) % 8 != 0)
        return SGQ_ERR_SHAPE;
    if (!gate || !up || !h)
        return SGQ_ERR_NULL;
    if (!aligned16(gate) || !aligned16(up) || !aligned16(h))
        return SGQ_ERR_ALIGN;
    int sms = current_device_sms();
    if (sms < 0)
        return sms;
    cudaError_t e = sgq::launch_glu(static_cast<const uint16_t *>(gate),
                                    static_cast<const uint16_t *>(up), static_cast<uint16_t *>(h),
                                    (long long)B * I, act, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SGQ_OK : fail_cuda(e);
}

} // extern "C"
