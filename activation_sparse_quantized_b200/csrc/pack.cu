// pack.cu -- group-wise asymmetric int4 quantization into the channel-major
// packed layout (version 1). Offline step, not on the timed path.
//
// Method: "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract
// (group-wise low-bit weight quantization, laid out so that the skipped input
// channels are skipped as whole runs of memory). The quantizer's details are
// this library's reading: 4 bits, asymmetric, groups of `group` consecutive
// input channels per output, the range always holding 0, fp16 scale
// s = RN((hi - lo) / 15), integer zero z = rint(-lo / s) in [0, 15],
// q = clamp(rint(w / s) + z, 0, 15), all in fp64 with IEEE division and
// round-half-to-even, so the result is fixed bit for bit.
#include "sgq_device.cuh"
#include "sgq_launch.h"

namespace sgq {

namespace {

struct GroupQuant {
    double s;       // scale as a double (exactly the fp16 value)
    double z;       // integer zero point
    uint32_t packed; // fp16 scale | fp16 zero << 16
    bool bad;
};

__device__ __forceinline__ double half_bits_to_double(uint16_t h)
{
    return (double)__half2float(__ushort_as_half(h));
}

// Range and parameters of one group of g weights of one output row.
__device__ GroupQuant quantize_group(const uint16_t *w, int g)
{
    double lo = 0.0, hi = 0.0;
    bool bad = false;
    for (int j = 0; j < g; j += 8) {
        uint4 v = *reinterpret_cast<const uint4 *>(w + j);
        const uint16_t *h = reinterpret_cast<const uint16_t *>(&v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            double d = half_bits_to_double(h[e]);
            if (!isfinite(d))
                bad = true;
            if (d < lo)
                lo = d;
            if (d > hi)
                hi = d;
        }
    }
    GroupQuant r;
    r.bad = bad;
    __half sh = __double2half((hi - lo) / 15.0);
    double sv = (double)__half2float(sh);
    double zv;
    if (bad || sv == 0.0) {
        sh = __ushort_as_half((uint16_t)0x3c00); // 1.0
        sv = 1.0;
        zv = 0.0;
    } else {
        zv = rint(-lo / sv);
        zv = zv <= 0.0 ? 0.0 : (zv > 15.0 ? 15.0 : zv); // -0 becomes +0
    }
    r.s = sv;
    r.z = zv;
    r.packed = (uint32_t)__half_as_ushort(sh) |
               ((uint32_t)__half_as_ushort(__double2half(zv)) << 16);
    return r;
}

__device__ __forceinline__ uint32_t code_of(uint16_t wbits, const GroupQuant &p)
{
    if (p.bad)
        return 0;
    double c = rint(half_bits_to_double(wbits) / p.s) + p.z;
    c = c <= 0.0 ? 0.0 : (c > 15.0 ? 15.0 : c);
    return (uint32_t)c;
}

// One thread per (output pair, group): outputs 2b and 2b+1 share the bytes
// of the packed rows. Consecutive threads take consecutive b, so the byte
// stores of one k are coalesced across a warp.
__global__ void pack_kernel(const uint16_t *__restrict__ W, int N, int K, int g,
                            uint8_t *__restrict__ qweight, uint32_t *__restrict__ sz,
                            int32_t *status)
{
    const int half_n = N / 2;
    const int G = K / g;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)half_n * G)
        return;
    const int b = (int)(t % half_n);
    const int grp = (int)(t / half_n);
    const uint16_t *w0 = W + (size_t)(2 * b) * K + (size_t)grp * g;
    const uint16_t *w1 = W + (size_t)(2 * b + 1) * K + (size_t)grp * g;
    GroupQuant p0 = quantize_group(w0, g);
    GroupQuant p1 = quantize_group(w1, g);
    if (p0.bad || p1.bad)
        set_status(status, SGQ_STATUS_NONFINITE_W);
    sz[(size_t)grp * N + 2 * b] = p0.packed;
    sz[(size_t)grp * N + 2 * b + 1] = p1.packed;
    for (int j = 0; j < g; ++j) {
        uint32_t c0 = code_of(w0[j], p0);
        uint32_t c1 = code_of(w1[j], p1);
        qweight[(size_t)(grp * g + j) * half_n + b] = (uint8_t)(c0 | (c1 << 4));
    }
}

} // namespace

cudaError_t launch_pack(const uint16_t *W, int N, int K, int g, uint8_t *qweight, uint32_t *sz,
                        int32_t *status, cudaStream_t stream)
{
    const long long threads = (long long)(N / 2) * (K / g);
    const int block = 128;
    const long long grid = (threads + block - 1) / block;
    pack_kernel<<<(unsigned)grid, block, 0, stream>>>(W, N, K, g, qweight, sz, status);
    return cudaGetLastError();
}

} // namespace sgq
