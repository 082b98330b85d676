// sgq_launch.h -- internal host-side launchers behind the C ABI (not exported).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sgq.h"

namespace sgq {

struct Thresholds {
    float t[SGQ_MAX_BATCH];
};

// Where the rows (active input channels) of a GEMV come from.
enum RowSource : int {
    ROWS_LIST = 0,   // device list idx[0..*count)
    ROWS_DENSE = 1,  // every channel
    ROWS_THRESH = 2, // |x[b][k]| > t_b for some row b, found by each CTA for its own channel slice
    ROWS_MASK = 3,   // bit k of a device bitmask, decoded by each CTA for its own slice
    ROWS_GLU = 4,    // x = bf16(act(gate) * up) from the fp32 sums of a gate/up GEMV, |x| > t
};

// What the epilogue writes from the fp32 sums of the N GEMV outputs.
enum Epilogue : int {
    EPI_PLAIN = 0,    // y[b][n] = bf16(sum[b][n])
    EPI_GLU_SILU = 1, // N = 2I stacked (gate; up): y[b][i] = bf16(SiLU(sum[b][i]) * sum[b][I + i])
    EPI_GLU_RELU = 2, // the same with ReLU
};

struct GemvProblem {
    const uint8_t *qweight;
    const uint32_t *sz;
    const uint16_t *x;
    const int32_t *idx;
    const int32_t *count;
    const uint32_t *mask; // ROWS_MASK: bit k % 32 of word k / 32 = channel k active
    const uint8_t *keep;  // 2:4 layout: keep nibbles [K/g][N/4] (NULL = dense layout)
    uint16_t *y;
    float *y_f32;
    float *ws_acc;
    int32_t *status;
    int N, K, group, B;
    float t;
    float tb[SGQ_MAX_BATCH]; // ROWS_THRESH at B > 1: threshold of each batch row
    int source;
    int epilogue; // Epilogue; y (and y_f32) are [B][N/2] for the GLU epilogues
    bool accumulate; // add into ws_acc (the caller's fp32 [B][N]) and launch no epilogue kernel
    // ROWS_GLU: gate = gu[k], up = gu[K + k] (fp32 sums, 2K floats), the activation,
    // and an optional bf16 copy of x = h written once per channel
    const float *gu;
    int glu_act;
    uint16_t *h_out;
    // the epilogue kernel also zeroes zero_extra[0 .. zero_extra_n) (consumed sums)
    float *zero_extra;
    int zero_extra_n;
    // test hook (tensor-core batch kernel): withhold the last run's "ready"
    // commit, so that the waits on it run out and set SGQ_STATUS_TIMEOUT
    int debug_withhold_ready;
};

// Bytes of workspace (partial sums + tile counters) for N outputs, B rows.
size_t gemv_workspace_bytes(int N, int B);

cudaError_t launch_pack(const uint16_t *W, int N, int K, int g, uint8_t *qweight, uint32_t *sz,
                        int32_t *status, cudaStream_t stream);
cudaError_t launch_pack_nm(const uint16_t *W, int N, int K, int g, uint8_t *qweight,
                           uint8_t *keep, uint32_t *sz, int32_t *status, cudaStream_t stream);
cudaError_t launch_select(const uint16_t *x, int B, int K, const Thresholds &th, int32_t *idx,
                          int32_t *count, cudaStream_t stream);
cudaError_t launch_select_mask(const uint16_t *x, int B, int K, const Thresholds &th,
                               uint32_t *mask, int32_t *count, cudaStream_t stream);
cudaError_t launch_gemv(const GemvProblem &p, int num_sms, cudaStream_t stream);
// B > 1 over the plain layout (gemv_mma.cu), then the split-K epilogue.
cudaError_t launch_gemv_mma(const GemvProblem &p, int num_sms, cudaStream_t stream);
// The split-K epilogue kernel alone (PDL-chained behind a GEMV grid).
cudaError_t launch_finalize(const GemvProblem &p, cudaStream_t stream);
// Records e as the last CUDA error of this thread; returns SGQ_ERR_CUDA.
int record_cuda_error(cudaError_t e);

cudaError_t launch_glu(const uint16_t *gate, const uint16_t *up, uint16_t *h, long long n,
                       int act, int num_sms, cudaStream_t stream);

} // namespace sgq
