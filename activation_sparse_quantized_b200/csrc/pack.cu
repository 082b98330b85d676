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

// 2:4 weight sparsity along the outputs of each channel row (the N:M
// sparsity of "SparseDecoding: Decoding-Aware Pruning for Accurate and
// Efficient LLM Inference", Abstract, placed so that it composes with
// skipping whole input channels). Per quantization group G and block of 4
// outputs, the 2 outputs with the largest sum of squared weights over the
// group are kept (ties to the lower output); the group's channels share that
// choice. Sums of squares of fp16 values are exact in fp64, so the choice is
// fixed bit for bit. Kept outputs are quantized as in the dense layout.
//
// Layout (N % 64 == 0): qweight u8 [K][N/4], byte j of row k = code of slot
// 2j | slot 2j+1 << 4, where slots 2j and 2j+1 are the kept outputs of block j
// in ascending order; keep u8 [K/g][N/8], byte j = keep nibble of block 2j |
// that of block 2j+1 << 4 (bit i = output 4 block + i kept); sz [K/g][N/2]
// (fp16 s, fp16 z) per slot. A block holding NaN/Inf keeps outputs 0 and 1
// with s = 1, z = 0, q = 0 and sets SGQ_STATUS_NONFINITE_W.
//
// One thread per (group, pair of blocks): it owns one keep byte and two bytes
// of each of the group's packed rows.
__global__ void pack_nm_kernel(const uint16_t *__restrict__ W, int N, int K, int g,
                               uint8_t *__restrict__ qweight, uint8_t *__restrict__ keep,
                               uint32_t *__restrict__ sz, int32_t *status)
{
    const int pairs = N / 8;
    const int G = K / g;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)pairs * G)
        return;
    const int jj = (int)(t % pairs);
    const int grp = (int)(t / pairs);
    uint32_t kbyte = 0;
    for (int h = 0; h < 2; ++h) {
        const int j = 2 * jj + h; // block: outputs 4j .. 4j + 3
        double e[4];
        bool bad = false;
        for (int i = 0; i < 4; ++i) {
            const uint16_t *w = W + (size_t)(4 * j + i) * K + (size_t)grp * g;
            double acc = 0.0;
            for (int r = 0; r < g; ++r) {
                const double d = half_bits_to_double(w[r]);
                if (!isfinite(d))
                    bad = true;
                acc = __dadd_rn(acc, __dmul_rn(d, d)); // no contraction: fixed rounding
            }
            e[i] = acc;
        }
        int a = 0, b = 1;
        if (!bad) {
            a = 0;
            for (int i = 1; i < 4; ++i)
                if (e[i] > e[a])
                    a = i;
            b = (a == 0) ? 1 : 0;
            for (int i = 0; i < 4; ++i)
                if (i != a && e[i] > e[b])
                    b = i;
            if (a > b) {
                const int tmp = a;
                a = b;
                b = tmp;
            }
        } else {
            set_status(status, SGQ_STATUS_NONFINITE_W);
        }
        kbyte |= ((1u << a) | (1u << b)) << (4 * h);
        GroupQuant p0, p1;
        if (bad) {
            p0.bad = p1.bad = true;
            p0.s = p1.s = 1.0;
            p0.z = p1.z = 0.0;
            p0.packed = p1.packed = 0x3c00u; // s = 1, z = +0
        } else {
            p0 = quantize_group(W + (size_t)(4 * j + a) * K + (size_t)grp * g, g);
            p1 = quantize_group(W + (size_t)(4 * j + b) * K + (size_t)grp * g, g);
        }
        sz[(size_t)grp * (N / 2) + 2 * j] = p0.packed;
        sz[(size_t)grp * (N / 2) + 2 * j + 1] = p1.packed;
        const uint16_t *w0 = W + (size_t)(4 * j + a) * K + (size_t)grp * g;
        const uint16_t *w1 = W + (size_t)(4 * j + b) * K + (size_t)grp * g;
        for (int r = 0; r < g; ++r) {
            const uint32_t c0 = code_of(w0[r], p0);
            const uint32_t c1 = code_of(w1[r], p1);
            qweight[(size_t)(grp * g + r) * (N / 4) + j] = (uint8_t)(c0 | (c1 << 4));
        }
    }
    keep[(size_t)grp * (N / 8) + jj] = (uint8_t)kbyte;
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

cudaError_t launch_pack_nm(const uint16_t *W, int N, int K, int g, uint8_t *qweight,
                           uint8_t *keep, uint32_t *sz, int32_t *status, cudaStream_t stream)
{
    const long long threads = (long long)(N / 8) * (K / g);
    const int block = 128;
    const long long grid = (threads + block - 1) / block;
    pack_nm_kernel<<<(unsigned)grid, block, 0, stream>>>(W, N, K, g, qweight, keep, sz, status);
    return cudaGetLastError();
}

} // namespace sgq
