// select.cu -- runtime gathering of the active channels.
//
// Method: "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract
// (a compact runtime mechanism that gathers the sparse indices). Channel k is
// active when |x[b][k]| > t[b] for some batch row b (strict, so t = 0 keeps
// exactly the nonzero channels, the ReLU zeros of "SVD Contextual Sparsity
// Predictors", Abstract). The list is written in ascending order.
//
// One CTA of 1024 threads walks the channels in tiles of 8 per thread:
// 16-byte loads of each batch row, a per-thread 8-bit mask, a warp shuffle
// scan and a cross-warp scan in shared memory, then each thread writes its
// indices at its exclusive offset. The activation vector is small (2*B*K
// bytes), so one CTA keeps the whole list ordered without any inter-CTA wait.
#include "sgq_device.cuh"
#include "sgq_launch.h"

namespace sgq {

namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t *__restrict__ x,
                                                             int B, int K, Thresholds th,
                                                             int32_t *__restrict__ idx,
                                                             int32_t *__restrict__ count)
{
    __shared__ int warp_excl[kSelWarps];
    __shared__ int tile_total;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    int offset = 0;
    for (int base = 0; base < K; base += 8 * kSelThreads) {
        const int c0 = base + tid * 8;
        uint32_t mask = 0;
        if (c0 < K) {
            for (int b = 0; b < B; ++b) {
                uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)b * K + c0));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const float t = th.t[b];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = fabsf(__uint_as_float(w[e] << 16));
                    float hi = fabsf(__uint_as_float(w[e] & 0xffff0000u));
                    mask |= (lo > t ? 1u : 0u) << (2 * e);
                    mask |= (hi > t ? 1u : 0u) << (2 * e + 1);
                }
            }
        }
        const int cnt = __popc(mask);
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d)
                incl += v;
        }
        if (lane == 31)
            warp_excl[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int wv = warp_excl[lane];
            int wi = wv;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                int v = __shfl_up_sync(0xffffffffu, wi, d);
                if (lane >= d)
                    wi += v;
            }
            warp_excl[lane] = wi - wv;
            if (lane == 31)
                tile_total = wi;
        }
        __syncthreads();
        int pos = offset + warp_excl[warp] + incl - cnt;
        while (mask) {
            const int j = __ffs(mask) - 1;
            idx[pos++] = c0 + j;
            mask &= mask - 1;
        }
        offset += tile_total;
        __syncthreads(); // warp_excl / tile_total are rewritten by the next tile
    }
    if (tid == 0)
        *count = offset;
}

// Bitmask form of the same active set, one bit per channel (the bitmask
// indexing of "SparseDecoding: Decoding-Aware Pruning for Accurate and
// Efficient LLM Inference", Abstract, and the shared-memory bitmap decoding of
// "Unified Static-Dynamic Pruning for Efficient LLM Inference", Abstract, in
// that page's similar-work list): bit k % 32 of word k / 32 is set when
// channel k is active. Each thread forms the 8-bit mask of its 8 channels as
// above; the lead lane of every 4 lanes gathers its neighbours' bytes with
// three shuffles and stores one 32-bit word. The CTA also reduces the count.
__global__ void __launch_bounds__(kSelThreads) select_mask_kernel(const uint16_t *__restrict__ x,
                                                                  int B, int K, Thresholds th,
                                                                  uint32_t *__restrict__ mask,
                                                                  int32_t *__restrict__ count)
{
    __shared__ int warp_cnt[kSelWarps];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    int total = 0;
    for (int base = 0; base < K; base += 8 * kSelThreads) {
        const int c0 = base + tid * 8;
        uint32_t m = 0;
        if (c0 < K) {
            for (int b = 0; b < B; ++b) {
                uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)b * K + c0));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const float t = th.t[b];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = fabsf(__uint_as_float(w[e] << 16));
                    float hi = fabsf(__uint_as_float(w[e] & 0xffff0000u));
                    m |= (lo > t ? 1u : 0u) << (2 * e);
                    m |= (hi > t ? 1u : 0u) << (2 * e + 1);
                }
            }
        }
        total += __popc(m);
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, m, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, m, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, m, 3);
        if ((lane & 3) == 0 && c0 < K)
            mask[c0 >> 5] = m | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1)
        total += __shfl_xor_sync(0xffffffffu, total, d);
    if (lane == 0)
        warp_cnt[warp] = total;
    __syncthreads();
    if (warp == 0) {
        int v = warp_cnt[lane];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1)
            v += __shfl_xor_sync(0xffffffffu, v, d);
        if (lane == 0 && count)
            *count = v;
    }
}

} // namespace

cudaError_t launch_select(const uint16_t *x, int B, int K, const Thresholds &th, int32_t *idx,
                          int32_t *count, cudaStream_t stream)
{
    select_kernel<<<1, kSelThreads, 0, stream>>>(x, B, K, th, idx, count);
    return cudaGetLastError();
}

cudaError_t launch_select_mask(const uint16_t *x, int B, int K, const Thresholds &th,
                               uint32_t *mask, int32_t *count, cudaStream_t stream)
{
    select_mask_kernel<<<1, kSelThreads, 0, stream>>>(x, B, K, th, mask, count);
    return cudaGetLastError();
}

} // namespace sgq
