// sgq_device.cuh -- device helpers shared by the libsgq kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/sgq.h"

namespace sgq {

// ---- asynchronous global -> shared copies (LDGSTS), per-thread groups ----

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte copy that bypasses L1 (weights are streamed once).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src)
                 : "memory");
}

__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// ---- L2 prefetch hints ----

// [p, p + bytes) into L2 with one bulk prefetch (p 16-byte aligned, bytes a
// multiple of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes)
{
    if (bytes)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// The 128-byte lines of [p, end) into L2, one line per lane of the calling
// warp (at most 32 lines).
__device__ __forceinline__ void prefetch_l2_lines(const void *p, const void *end)
{
    const uintptr_t a = (uintptr_t)p & ~(uintptr_t)127, e = (uintptr_t)end;
    const uintptr_t line = a + 128u * (threadIdx.x & 31);
    if (line < e)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(line) : "memory");
}

// ---- Programmatic dependent launch ----

__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

__device__ __forceinline__ void grid_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---- arithmetic ----

// d = a * b + c on two fp32 lanes at once (sm_100 packed FMA), round to
// nearest, subnormals kept (no .ftz).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Exact power of two 2^e as an fp32 for e in [-126, 127].
__device__ __forceinline__ float pow2f(int e)
{
    return __uint_as_float((uint32_t)(e + 127) << 23);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b)
{
    return __uint_as_float((uint32_t)b << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float v)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ---- global reductions / cache-bypassing accesses ----

__device__ __forceinline__ void red_add_v4(float *gptr, float4 v)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(gptr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ float4 ld_cg_v4(const float *gptr)
{
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];\n"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(gptr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_cg_f32(const float *gptr)
{
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];\n" : "=f"(v) : "l"(gptr) : "memory");
    return v;
}

__device__ __forceinline__ void st_cg_v4(float *gptr, float4 v)
{
    asm volatile("st.global.cg.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(gptr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ void set_status(int32_t *status, int32_t bits)
{
    if (status)
        atomicOr(status, bits);
}

// Gated activation act(g) * u in fp32: SiLU g / (1 + e^-g) (Llama / Qwen
// FFNs) or ReLU max(g, 0) (the ReGLU FFNs of "SVD Contextual Sparsity
// Predictors for Fast LLM Inference", Abstract, whose zeros the down
// projection then skips).
template <int ACT>
__device__ __forceinline__ float act_mul(float g, float u)
{
    float a;
    if (ACT == SGQ_ACT_SILU)
        a = g / (1.0f + expf(-g));
    else
        a = g > 0.0f ? g : 0.0f;
    return a * u;
}

} // namespace sgq
