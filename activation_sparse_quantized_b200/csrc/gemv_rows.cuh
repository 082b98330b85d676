// gemv_rows.cuh -- pieces shared by the GEMV kernels (gemv.cu, gemv_mma.cu):
// the per-launch parameters, the row lists of a CTA (its share of the active
// channels: an index list, a dense range, a bitmask or a threshold on x) and
// the launch helper with programmatic dependent launch.
//
// Method: "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract:
// the active channels are gathered at run time into a compact index list,
// and only their weight runs are read.
#pragma once

#include "sgq_device.cuh"
#include "sgq_launch.h"

namespace sgq {

namespace {

constexpr int kTileN1 = 1024;            // B = 1: outputs per tile, 32 per lane
constexpr int kRowBytes1 = kTileN1 / 2;  // bytes of one packed row per tile

struct KParams {
    GemvProblem p;
    int n_tiles;
    int k_splits;
    int rows_cap;  // capacity of the per-CTA row arrays
    int span_cap;  // groups of scale/zero staged in shared memory per CTA
    int lg;        // log2(group)
    int nb;        // batch groups of warps (1 for B = 1)
    int stages;    // tensor-core kernel: operand stages in shared memory
    int bp;        // tensor-core kernel: batch columns of the staged x (B padded)
};

__device__ __forceinline__ int warp_max_exponent(float m)
{
#pragma unroll
    for (int d = 16; d > 0; d >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (!(m > 0.0f) || isinf(m))
        return INT32_MIN; // all zero (or non-finite): no scaling
    return ilogbf(m);
}

// Exclusive prefix, over runs, of the per-run counts in scan[] for the runs
// 32c .. 32c + 31 (one per lane), plus the carry from the earlier chunks: a
// warp scan instead of a serial walk over shared memory. Returns the lane's
// exclusive prefix; *chunk_total receives the chunk's sum (every lane).
__device__ __forceinline__ int chunk_prefix(const int *scan, int runs, int c, int carry,
                                            int *chunk_total)
{
    const int lane = threadIdx.x & 31;
    const int r = c * 32 + lane;
    const int v = (r < runs) ? scan[r] : 0;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d)
            incl += t;
    }
    *chunk_total = __shfl_sync(0xffffffffu, incl, 31);
    return carry + incl - v;
}

// Channel slice [c0, c1) of split s when channels are dealt out in runs of 8.
__device__ __forceinline__ void channel_slice(const KParams &kp, int split, int &c0, int &c1)
{
    const int K8 = kp.p.K / 8;
    c0 = (int)((long long)K8 * split / kp.k_splits) * 8;
    c1 = (int)((long long)K8 * (split + 1) / kp.k_splits) * 8;
}

// ---------------------------------------------------------------------------
// Row lists: fill ridx[0..nr) (and rx = x for ROWS_THRESH) for this CTA and
// return nr. Entries outside [0, K) become -1 (their x is 0; they read row 0).
// Must be called by all threads; ends with a barrier.
// ---------------------------------------------------------------------------
template <int SRC, int NT, bool FILL_X = false>
__device__ int build_rows(const KParams &kp, int split, int32_t *ridx, float *rx, int *scan,
                          float *xs = nullptr, bool write_h = false, int list_lo = -1,
                          int list_hi = -1)
{
    const GemvProblem &p = kp.p;
    const int tid = threadIdx.x;
    if (SRC == ROWS_LIST) {
        // entries [list_lo, list_hi) when given (the caller has checked the
        // count), else this split's share of the list
        int r0 = list_lo, r1 = list_hi;
        if (list_lo < 0) {
            const int c = __ldg(p.count);
            const int a = c < 0 ? 0 : (c > p.K ? p.K : c);
            if (a != c && tid == 0 && blockIdx.x == 0)
                set_status(p.status, SGQ_STATUS_BAD_COUNT);
            r0 = (int)((long long)a * split / kp.k_splits);
            r1 = (int)((long long)a * (split + 1) / kp.k_splits);
        }
        for (int j = tid; j < r1 - r0; j += NT) {
            int k = __ldg(p.idx + r0 + j);
            if ((unsigned)k >= (unsigned)p.K) {
                set_status(p.status, SGQ_STATUS_BAD_INDEX);
                k = -1;
            }
            ridx[j] = k;
        }
        __syncthreads();
        return r1 - r0;
    } else if (SRC == ROWS_DENSE) {
        const int r0 = (int)((long long)p.K * split / kp.k_splits);
        const int r1 = (int)((long long)p.K * (split + 1) / kp.k_splits);
        for (int j = tid; j < r1 - r0; j += NT)
            ridx[j] = r0 + j;
        __syncthreads();
        return r1 - r0;
    } else if (SRC == ROWS_MASK) {
        // Decode this CTA's channel slice of the bitmask: runs of 32 channels,
        // one per lane, a ballot per run, the count of each run in scan[]; a
        // second pass recomputes the ballots (the mask words stay in L1) and
        // writes each active channel at its ascending position. With FILL_X
        // (batch 1) the first pass also reads the slice of x, coalesced and
        // alongside the mask words, into xs[], and the second copies the x of
        // each active channel into rx[].
        int c0, c1;
        channel_slice(kp, split, c0, c1);
        const int lane = tid & 31, warp = tid >> 5;
        const int runs = (c1 - c0 + 31) / 32;
        auto run_bits = [&](int q) -> uint32_t {
            const int c = c0 + q * 32 + lane;
            const bool act = (c < c1) && ((__ldg(p.mask + (c >> 5)) >> (c & 31)) & 1u);
            return __ballot_sync(0xffffffffu, act);
        };
        for (int q = warp; q < runs; q += NT / 32) {
            if (FILL_X) {
                const int c = c0 + q * 32 + lane;
                if (c < c1)
                    xs[c - c0] = bf16_bits_to_float(__ldg(p.x + c));
            }
            const uint32_t m = run_bits(q);
            if (lane == 0)
                scan[q] = __popc(m);
        }
        __syncthreads();
        int total = 0;
        for (int c = 0; c * 32 < runs; ++c) {
            int ct;
            const int excl = chunk_prefix(scan, runs, c, total, &ct);
            // this warp's runs in the chunk (q is warp-uniform)
            for (int q = c * 32 + ((warp - c * 32) % (NT / 32) + NT / 32) % (NT / 32);
                 q < runs && q < c * 32 + 32; q += NT / 32) {
                const int base = __shfl_sync(0xffffffffu, excl, q - c * 32);
                const uint32_t m = run_bits(q);
                if ((m >> lane) & 1u) {
                    const int pos = base + __popc(m & ((1u << lane) - 1u));
                    ridx[pos] = c0 + q * 32 + lane;
                    if (FILL_X)
                        rx[pos] = xs[q * 32 + lane];
                }
            }
            total += ct;
        }
        __syncthreads();
        return total;
    } else if (SRC == ROWS_THRESH && !FILL_X) {
        // Batch rows (B > 1): channel c of this CTA's slice is active when
        // |x[b][c]| > t_b for some row b (the union of the rows' active sets).
        // Runs of 32 channels, one per lane, a ballot per run and the count of
        // each run in scan[]; a second pass recomputes the ballots (the x lines
        // stay in L1) and writes each active channel at its ascending position.
        // Channels [8 list_lo, 8 list_hi) when given (a segment), else this
        // split's slice.
        int c0, c1;
        if (list_lo >= 0) {
            c0 = 8 * list_lo;
            c1 = 8 * list_hi;
        } else {
            channel_slice(kp, split, c0, c1);
        }
        const int lane = tid & 31, warp = tid >> 5;
        const int runs = (c1 - c0 + 31) / 32;
        auto run_bits = [&](int q) -> uint32_t {
            const int c = c0 + q * 32 + lane;
            bool act = false;
            if (c < c1)
                for (int b = 0; b < p.B; ++b)
                    act |= (fabsf(bf16_bits_to_float(__ldg(p.x + (size_t)b * p.K + c))) >
                                  p.tb[b]);
            return __ballot_sync(0xffffffffu, act);
        };
        for (int q = warp; q < runs; q += NT / 32) {
            const uint32_t m = run_bits(q);
            if (lane == 0)
                scan[q] = __popc(m);
        }
        __syncthreads();
        int total = 0;
        for (int c = 0; c * 32 < runs; ++c) {
            int ct;
            const int excl = chunk_prefix(scan, runs, c, total, &ct);
            for (int q = c * 32 + ((warp - c * 32) % (NT / 32) + NT / 32) % (NT / 32);
                 q < runs && q < c * 32 + 32; q += NT / 32) {
                const int base = __shfl_sync(0xffffffffu, excl, q - c * 32);
                const uint32_t m = run_bits(q);
                if ((m >> lane) & 1u)
                    ridx[base + __popc(m & ((1u << lane) - 1u))] = c0 + q * 32 + lane;
            }
            total += ct;
        }
        __syncthreads();
        return total;
    } else {
        // Threshold this CTA's channel slice: each warp takes runs of 32
        // channels, one per lane; a ballot gives each run's active channels,
        // a count per run and a prefix over runs give the ascending positions.
        int c0, c1;
        channel_slice(kp, split, c0, c1);
        const int lane = tid & 31, warp = tid >> 5;
        const int runs = (c1 - c0 + 31) / 32;
        uint32_t mask[4];
        float xv[4];
        // Runs of this warp: warp, warp + NT/32, ... (the launcher keeps
        // runs <= 4 * NT / 32).
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int q = warp + u * (NT / 32);
            const int c = c0 + q * 32 + lane;
            float v = 0.f;
            bool act = false;
            if (q < runs && c < c1) {
                if (SRC == ROWS_GLU) {
                    // x = h = bf16(act(gate) * up) from the consumed fp32 sums
                    // (written by the previous kernel's reductions: read from L2)
                    const float gt = ld_cg_f32(p.gu + c), up = ld_cg_f32(p.gu + p.K + c);
                    const float hv = (p.glu_act == SGQ_ACT_SILU) ? act_mul<SGQ_ACT_SILU>(gt, up)
                                                                 : act_mul<SGQ_ACT_RELU>(gt, up);
                    const uint16_t hb = float_to_bf16_bits(hv);
                    if (write_h && p.h_out)
                        p.h_out[c] = hb;
                    v = bf16_bits_to_float(hb);
                } else {
                    v = bf16_bits_to_float(__ldg(p.x + c));
                }
                act = fabsf(v) > p.t;
            }
            mask[u] = __ballot_sync(0xffffffffu, act);
            xv[u] = v;
            if (lane == 0 && q < runs)
                scan[q] = __popc(mask[u]);
        }
        __syncthreads();
        // runs <= 4 * NT / 32 <= 32 (the launcher keeps it so): one chunk
        int total;
        const int excl = chunk_prefix(scan, runs, 0, 0, &total);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int q = warp + u * (NT / 32); // warp-uniform
            if (q < runs) {
                const int base = __shfl_sync(0xffffffffu, excl, q);
                if ((mask[u] >> lane) & 1u) {
                    const int pos = base + __popc(mask[u] & ((1u << lane) - 1u));
                    ridx[pos] = c0 + q * 32 + lane;
                    rx[pos] = xv[u];
                }
            }
        }
        __syncthreads();
        return total;
    }
}

constexpr size_t kMaxSmem = 227 * 1024;

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

template <typename Kern, typename Arg>
cudaError_t launch_pdl(Kern kern, int grid, int block, size_t smem, cudaStream_t stream,
                       const Arg &arg)
{
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess)
            return err;
    }
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
    return cudaLaunchKernelEx(&cfg, kern, arg);
}

} // namespace

} // namespace sgq
