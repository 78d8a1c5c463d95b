// common.cuh -- small device helpers shared by the SSD kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mamba_ssd.h"

namespace ssd {

constexpr float kLog2e = 1.4426950408889634f;

// Storage types of activations.
template <typename T> struct Store;
template <> struct Store<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ float ldg(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ float from(float v) { return v; }
};
template <> struct Store<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ float ldg(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ __nv_bfloat16 from(float v) { return __float2bfloat16_rn(v); }
};

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// softplus(z) = log(1 + e^z), evaluated without overflow for large z.
__device__ __forceinline__ float softplus_f(float z) {
    return z > 20.f ? z + log1pf(expf(-z)) : log1pf(expf(z));
}

// dt = clip(softplus(dt_raw + bias), dt_min, dt_max)
__device__ __forceinline__ float discretise_dt(float raw, float bias, float dt_min, float dt_max) {
    return fminf(fmaxf(softplus_f(raw + bias), dt_min), dt_max);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// SiLU with the fast hardware exponential and division, for the streaming kernels where the
// IEEE forms cost more issue slots than the memory traffic leaves (relative error about 1e-6,
// far below a bf16 rounding).  The exponent is clamped at 80 so that 1 + e^-z stays below
// 2^126, where __fdividef is accurate to a few ulp; below z = -80 the result is 0 to within
// 1e-33.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.f + __expf(fminf(-z, 80.f))); }

// Inclusive warp scan (sum) of one value per lane.
__device__ __forceinline__ float warp_inclusive_sum(float v) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float n = __shfl_up_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) >= o) v += n;
    }
    return v;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization
// may start while the kernel before it in the stream is still running; grid_dependency_wait()
// blocks the calling thread until that kernel has completed and its memory operations are
// visible (a no-op for an ordinary launch), so every global access comes after it.
// allow_dependents() lets the next such kernel be scheduled once every CTA of this grid has
// called it (or exited).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// after_wait(p): p, re-derived through an empty volatile asm placed after grid_dependency_wait().
// A __restrict__ kernel parameter tells the compiler that nothing else writes its memory while
// the kernel runs, which lets it move loads and stores through that pointer above the wait's
// asm (the asm's memory clobber does not cover a pointer that never escaped) -- exactly wrong
// when the previous kernel is still writing that memory.  An access through the returned
// pointer depends on an asm that comes after the wait, so it cannot move above it.  Every
// raw pointer a PDL kernel touches after its wait goes through this.
template <typename T>
__device__ __forceinline__ T *after_wait(T *p) {
    asm volatile("" : "+l"(p));
    return p;
}

// Drop the 128-byte L2 line at p (128-byte aligned) without writing it back: for a workspace
// intermediate whose last read has happened (by every thread that reads it, in a happens-before
// order), so that its dirty line never costs a DRAM write.  The line's contents become
// undefined.
__device__ __forceinline__ void discard_l2_line(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// 16-byte L2-only load / global store with an L2 eviction-priority policy (a createpolicy result).
__device__ __forceinline__ float4 ldcg_hint(const float4 *p, uint64_t policy) {
    float4 v;
    asm volatile("ld.global.cg.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}
__device__ __forceinline__ void st_global_hint_v4(float4 *p, float4 v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w), "l"(policy)
                 : "memory");
}

// A global load with an L2 eviction-priority policy (a createpolicy result).
__device__ __forceinline__ float4 ld_global_hint(const float4 *p, uint64_t policy) {
    float4 v;
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

__host__ __device__ constexpr inline int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ constexpr inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace ssd
