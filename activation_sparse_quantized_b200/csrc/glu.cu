// glu.cu -- gated FFN activation h = act(gate) * up between the gate/up and
// the down projections. ReLU gating (the ReGLU FFNs of "SVD Contextual
// Sparsity Predictors for Fast LLM Inference", Abstract) produces the exact
// zeros that the down projection then skips; SiLU gating is the Llama / Qwen
// FFN. fp32 arithmetic, bf16 round-to-nearest-even output.
#include "sgq_device.cuh"
#include "sgq_launch.h"

namespace sgq {

namespace {

template <int ACT>
__global__ void glu_kernel(const uint4 *__restrict__ gate, const uint4 *__restrict__ up,
                           uint4 *__restrict__ h, long long nvec)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
         i += (long long)gridDim.x * blockDim.x) {
        uint4 gv = __ldg(gate + i), uv = __ldg(up + i);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t hw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float lo = act_mul<ACT>(__uint_as_float(gw[e] << 16), __uint_as_float(uw[e] << 16));
            float hi = act_mul<ACT>(__uint_as_float(gw[e] & 0xffff0000u),
                                    __uint_as_float(uw[e] & 0xffff0000u));
            hw[e] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
        }
        h[i] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
}

} // namespace

cudaError_t launch_glu(const uint16_t *gate, const uint16_t *up, uint16_t *h, long long n,
                       int act, int num_sms, cudaStream_t stream)
{
    const long long nvec = n / 8;
    const int block = 256;
    long long grid = (nvec + block - 1) / block;
    if (grid > (long long)num_sms * 8)
        grid = (long long)num_sms * 8;
    if (grid < 1)
        grid = 1;
    const uint4 *g4 = reinterpret_cast<const uint4 *>(gate);
    const uint4 *u4 = reinterpret_cast<const uint4 *>(up);
    uint4 *h4 = reinterpret_cast<uint4 *>(h);
    if (act == SGQ_ACT_SILU)
        glu_kernel<SGQ_ACT_SILU><<<(unsigned)grid, block, 0, stream>>>(g4, u4, h4, nvec);
    else
        glu_kernel<SGQ_ACT_RELU><<<(unsigned)grid, block, 0, stream>>>(g4, u4, h4, nvec);
    return cudaGetLastError();
}

} // namespace sgq
