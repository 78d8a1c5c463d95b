// stream.cuh -- helpers of the CUDA-core streaming kernels (the gated norm's streaming forms):
// per-thread cp.async copies into a shared-memory ring, and a SiLU built on the flush-to-zero
// approximate base-2 exponential and reciprocal.
//
// cp.async is the asynchronous 16-byte global -> shared copy of the PTX ISA.  A thread's copies
// are grouped by cp.async.commit_group, and cp.async.wait_group N returns once at most N of the
// thread's most recent groups are still in flight; the copies it waited for are then visible
// to that thread (to the rest of the CTA after a barrier).  The wait is a hardware wait on the
// thread's own copies, not a spin on memory another agent writes.
#pragma once

#include <stdint.h>

namespace ssd {

// 16 bytes, global -> shared, with an L2 eviction policy (createpolicy)
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint64_t policy) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// SiLU(z) = z / (1 + e^-z), with e^-z taken as 2^(-z log2 e) by the PTX approximate base-2
// exponential and the division as a product with the approximate reciprocal, both in their
// flush-to-zero forms (the build keeps denormals, and the non-flushing forms of those
// instructions cost extra fix-up instructions per element).  Relative error about 2^-21;
// a denormal z counts as zero.  -z is capped at 80 so that 1 + e^-z stays finite.
__device__ __forceinline__ float silu_ftz(float z) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(fminf(-z, 80.f) * 1.4426950408889634f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
    return z * r;
}

}  // namespace ssd
