// select.cu -- runtime gathering of the active channels.
//
// Method: "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract
// (a compact runtime mechanism that gathers the sparse indices). Channel k is
// active when |x[b][k]| > t[b] for some batch row b (strict, so t = 0 keeps
// exactly the nonzero channels, the ReLU zeros of "SVD Contextual Sparsity
// Predictors", Abstract). The list is written in ascending order.
//
// Batch 1: tiles of 2048 channels, one CTA of 256 threads
// per tile, one 16-byte load (8 channels) per thread. A CTA finds where its
// indices start by counting the active channels of every earlier tile itself
// (at most 2 K bytes of x, from L2), so the list comes out in ascending order
// with no wait between CTAs and no scratch memory; the last CTA writes the
// count.
//
// Otherwise one CTA of 1024 threads walks the channels in tiles of 16 per
// thread: 16-byte loads of each batch row, a per-thread 16-bit mask, a warp
// shuffle scan and a cross-warp scan in shared memory; each thread puts its
// indices at its exclusive offset in a shared-memory copy of the tile, which
// the CTA then writes out with coalesced stores.
//
// Both are launched with programmatic dependent launch: they wait for the
// previous kernel only before reading x, and let the next one (the GEMV)
// launch early.
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
    extern __shared__ int s_idx[]; // one tile's indices, written out coalesced
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    grid_launch_dependents();
    grid_dependency_wait(); // x may come from the previous kernel
    int offset = 0;
    // tiles of 16 channels per thread: two 16-byte loads per batch row, both
    // in flight before either is used (K <= 16384 is a single tile)
    for (int base = 0; base < K; base += 16 * kSelThreads) {
        const int c0 = base + tid * 16;
        uint32_t mask = 0;
        for (int b = 0; b < B; ++b) {
            uint4 v[2];
#pragma unroll
            for (int h = 0; h < 2; ++h)
                v[h] = (c0 + 8 * h < K)
                           ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)b * K + c0 + 8 * h))
                           : make_uint4(0u, 0u, 0u, 0u);
            const float t = th.t[b];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (c0 + 8 * h >= K)
                    continue;
                const uint32_t w[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = fabsf(__uint_as_float(w[e] << 16));
                    float hi = fabsf(__uint_as_float(w[e] & 0xffff0000u));
                    mask |= (lo > t ? 1u : 0u) << (8 * h + 2 * e);
                    mask |= (hi > t ? 1u : 0u) << (8 * h + 2 * e + 1);
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
        int pos = warp_excl[warp] + incl - cnt; // position inside the tile
        while (mask) {
            const int j = __ffs(mask) - 1;
            s_idx[pos++] = c0 + j;
            mask &= mask - 1;
        }
        __syncthreads();
        const int tt = tile_total;
        for (int i = tid; i < tt; i += kSelThreads)
            idx[offset + i] = s_idx[i];
        offset += tt;
        __syncthreads(); // warp_excl / tile_total / s_idx are rewritten by the next tile
    }
    if (tid == 0)
        *count = offset;
}

constexpr int kTileThreads = 256;           // batch-1 tiled select: threads per CTA
constexpr int kTileCh = 8 * kTileThreads;   // channels per tile

// Active bits of 8 channels (one 16-byte load of bf16 x) against t.
__device__ __forceinline__ uint32_t mask8(const uint4 v, float t)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        m |= (fabsf(__uint_as_float(w[e] << 16)) > t ? 1u : 0u) << (2 * e);
        m |= (fabsf(__uint_as_float(w[e] & 0xffff0000u)) > t ? 1u : 0u) << (2 * e + 1);
    }
    return m;
}

// Batch 1: CTA c owns channels [c kTileCh, (c + 1) kTileCh).
__global__ void __launch_bounds__(kTileThreads) select_tiled_kernel(const uint16_t *__restrict__ x,
                                                                    int K, float t,
                                                                    int32_t *__restrict__ idx,
                                                                    int32_t *__restrict__ count)
{
    __shared__ int warp_sum[kTileThreads / 32], warp_excl[kTileThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lo = blockIdx.x * kTileCh;
    grid_launch_dependents();
    grid_dependency_wait(); // x may come from the previous kernel
    // this thread's 8 channels (issued first), then the earlier tiles' chunks
    const int c8 = lo / 8 + tid;
    const uint4 own = (8 * c8 < K) ? __ldg(reinterpret_cast<const uint4 *>(x) + c8)
                                   : make_uint4(0u, 0u, 0u, 0u);
    int before = 0;
    for (int ch = tid; ch < lo / 8; ch += kTileThreads)
        before += __popc(mask8(__ldg(reinterpret_cast<const uint4 *>(x) + ch), t));
    const uint32_t m = (8 * c8 < K) ? mask8(own, t) : 0u;
    const int cnt = __popc(m);
    // warp sums of `before` and inclusive warp scans of `cnt`
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d)
            incl += v;
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1)
        before += __shfl_xor_sync(0xffffffffu, before, d);
    if (lane == 31)
        warp_excl[warp] = incl;
    if (lane == 0)
        warp_sum[warp] = before;
    __syncthreads();
    int base = 0, wex = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kTileThreads / 32; ++w) {
        base += warp_sum[w];
        wex += (w < warp) ? warp_excl[w] : 0;
        total += warp_excl[w];
    }
    int pos = base + wex + incl - cnt;
    uint32_t mm = m;
    while (mm) {
        const int j = __ffs(mm) - 1;
        idx[pos++] = lo + 8 * tid + j;
        mm &= mm - 1;
    }
    if (blockIdx.x == gridDim.x - 1 && tid == 0)
        *count = base + total;
}

// Bitmask form of the same active set, one bit per channel (the bitmask
// indexing of "SparseDecoding: Decoding-Aware Pruning for Accurate and
// Efficient LLM Inference", Abstract, and the shared-memory bitmap decoding of
// "Unified Static-Dynamic Pruning for Efficient LLM Inference", Abstract, in
// that page's similar-work list): bit k % 32 of word k / 32 is set when
// channel k is active. Each thread forms the 16-bit mask of its 16 channels as
// above; the even lane of every pair takes its neighbour's half with one
// shuffle and stores one 32-bit word. The CTA also reduces the count.
__global__ void __launch_bounds__(kSelThreads) select_mask_kernel(const uint16_t *__restrict__ x,
                                                                  int B, int K, Thresholds th,
                                                                  uint32_t *__restrict__ mask,
                                                                  int32_t *__restrict__ count)
{
    __shared__ int warp_cnt[kSelWarps];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    grid_launch_dependents();
    grid_dependency_wait(); // x may come from the previous kernel
    int total = 0;
    for (int base = 0; base < K; base += 16 * kSelThreads) {
        const int c0 = base + tid * 16;
        uint32_t m = 0;
        for (int b = 0; b < B; ++b) {
            uint4 v[2];
#pragma unroll
            for (int h = 0; h < 2; ++h)
                v[h] = (c0 + 8 * h < K)
                           ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)b * K + c0 + 8 * h))
                           : make_uint4(0u, 0u, 0u, 0u);
            const float t = th.t[b];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (c0 + 8 * h >= K)
                    continue;
                const uint32_t w[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = fabsf(__uint_as_float(w[e] << 16));
                    float hi = fabsf(__uint_as_float(w[e] & 0xffff0000u));
                    m |= (lo > t ? 1u : 0u) << (8 * h + 2 * e);
                    m |= (hi > t ? 1u : 0u) << (8 * h + 2 * e + 1);
                }
            }
        }
        total += __popc(m);
        const uint32_t m1 = __shfl_down_sync(0xffffffffu, m, 1);
        if ((lane & 1) == 0 && c0 < K)
            mask[c0 >> 5] = m | (m1 << 16);
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

// One launch with programmatic dependent launch allowed.
template <typename Kern, typename... Args>
cudaError_t launch_pdl_sel(Kern kern, int grid, int block, size_t smem, cudaStream_t stream,
                           Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_select(const uint16_t *x, int B, int K, const Thresholds &th, int32_t *idx,
                          int32_t *count, cudaStream_t stream)
{
    if (B == 1 && K % 8 == 0)
        return launch_pdl_sel(select_tiled_kernel, (K + kTileCh - 1) / kTileCh, kTileThreads, 0,
                              stream, x, K, th.t[0], idx, count);
    const size_t smem = sizeof(int) * 16 * kSelThreads; // 64 KB: one tile of indices
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl_sel(select_kernel, 1, kSelThreads, smem, stream, x, B, K, th, idx, count);
}

cudaError_t launch_select_mask(const uint16_t *x, int B, int K, const Thresholds &th,
                               uint32_t *mask, int32_t *count, cudaStream_t stream)
{
    return launch_pdl_sel(select_mask_kernel, 1, kSelThreads, 0, stream, x, B, K, th, mask, count);
}

} // namespace sgq
