// Shared device helpers of libmep (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mep.h"   // the MEP_DERR_* bits the kernels set

namespace mep {

// Sticky per-device word of data errors (MEP_DERR_* bits), read by mep_get_error.
__device__ int32_t g_error_word;

__device__ __forceinline__ void flag_error(int32_t bit) { atomicOr(&g_error_word, bit); }

// Clears the given bits of the error word (the ones a reader has just reported).
__global__ void k_clear_error_bits(int32_t bits) { atomicAnd(&g_error_word, ~bits); }

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte global load that bypasses L1 allocation (read-once streams).
__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte global store.
__device__ __forceinline__ void st_v4(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// bf16 bits -> fp32 (exact: the bf16 bits are the high half of the fp32 bits).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2 (low half = a), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// bf16(p), round to nearest even, as an fp32 value: the packed conversion with a zero
// low half leaves the bf16 bits in the high half, which read as fp32 are that value.
__device__ __forceinline__ float round_bf16(float p) { return __uint_as_float(pack_bf16x2(0.0f, p)); }

// Two binary32 additions / multiplications in one instruction (sm_100 packed f32x2),
// each rounded to nearest even on its own: the same results as __fadd_rn / __fmul_rn
// on each half. Use them only where no packed multiply feeds an addition: such a pair
// can be fused into one rounding.
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b)
{
    float2 d;
    asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
        " add.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}\n"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b)
{
    float2 d;
    asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
        " mul.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}\n"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b)
{
    float2 d;
    asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
        " sub.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}\n"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Two fused multiply-adds a * b + c, each rounded once (to nearest even).
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n .reg .b64 pa, pb, pc, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
        " mov.b64 pc, {%6, %7};\n fma.rn.f32x2 pd, pa, pb, pc;\n mov.b64 {%0, %1}, pd;\n}\n"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// The largest of three floats in one instruction (sm_100 three-input max.f32): for
// inputs that are not NaN, fmaxf(fmaxf(a, b), c).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Programmatic dependent launch (the host launches the routing step's kernels with the
// programmatic-serialization attribute): pdl_wait() returns once the grid this one
// depends on has finished and its memory is visible (at once when there is none), so a
// kernel calls it before touching any memory the previous kernel may use;
// pdl_launch_dependents() lets the next kernel's CTAs be scheduled while this one runs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace mep
