// tmap.h -- TMA tensor-map creation (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// A 3-D bf16 tensor map with 128-byte swizzle and zero fill outside the tensor:
// dims (innermost first) d0, d1, d2; byte strides of dims 1 and 2; box box0 x box1 x box2
// (box0 * 2 bytes must be <= 128 for the swizzle).
cudaError_t make_tmap_bf16_3d(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                              uint32_t box0, uint32_t box1, uint32_t box2);

// The same with 64-byte swizzle (box0 * 2 bytes must be <= 64).
cudaError_t make_tmap_bf16_3d_sw64(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                                   uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                                   uint32_t box2);

// A 2-D bf16 tensor map with 128-byte swizzle: dims d0 (inner), d1; byte stride of dim 1.
cudaError_t make_tmap_bf16_2d(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1,
                              uint64_t stride1_bytes, uint32_t box0, uint32_t box1);

// A 2-D fp32 tensor map with 128-byte swizzle: dims d0 (inner), d1; byte stride of dim 1
// (box0 * 4 bytes must be <= 128 for the swizzle).
cudaError_t make_tmap_f32_2d(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1,
                             uint64_t stride1_bytes, uint32_t box0, uint32_t box1);

}  // namespace ssd
