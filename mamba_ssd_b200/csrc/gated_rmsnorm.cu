// gated_rmsnorm.cu -- the block step after the scan: y * SiLU(z), RMS-normalised per token
// and norm group, scaled per channel.
//
//   g   = y * SiLU(z)
//   out = g / sqrt(mean over the group's channels of g^2 + eps) * w
//
// Source: the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §4.1 (a norm takes its
// variance in float32 even for bf16 inputs) and §3.2 (norms sit next to the SSD and are fused
// into their neighbours); the gate and the per-group RMS are the Mamba-2 block's norm, which
// the pages name but do not spell out.
//
// One CTA per (token, norm group).  The group's GS channels stream in once as 16-byte vectors
// of y and z; each thread keeps its gated values in shared memory (fp32) and adds up their
// squares in fp32; the CTA reduces the sum, and a second pass over shared memory scales by the
// reciprocal RMS and by w and streams the result out.  HBM-bound: 3 * GS * sizeof(T) bytes per
// row (plus w, which stays in L2).  No waits of any kind.
#include "common.cuh"
#include "launch.h"

namespace ssd {

constexpr int kNormThreads = 256;
constexpr int kNormMaxGroup = 32768;  // channels per norm group: 128 KB of staged fp32
constexpr int kNormBatch = 3;         // 16-byte vectors of y and of z in flight per thread

template <typename T>
struct Vec16;  // 16 bytes of T
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
};
template <>
struct Vec16<float> {
    static constexpr int n = 4;
};

template <typename T>
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(const T *__restrict__ y,
                                                                     const T *__restrict__ z,
                                                                     const float *__restrict__ w,
                                                                     T *__restrict__ out, int C, int GS,
                                                                     float eps) {
    extern __shared__ __align__(16) float g_s[];  // [GS] gated values of this row
    __shared__ float red[kNormThreads / 32];
    constexpr int VEC = Vec16<T>::n;

    grid_dependency_wait();  // y comes from the kernel before
    y = after_wait(y);
    z = after_wait(z);
    w = after_wait(w);
    out = after_wait(out);

    const size_t base = (size_t)blockIdx.x * C + (size_t)blockIdx.y * GS;
    const int nvec = GS / VEC;
    const uint4 *y4 = reinterpret_cast<const uint4 *>(y + base);
    const uint4 *z4 = reinterpret_cast<const uint4 *>(z + base);

    // ---- pass 1: gate, stage, sum of squares (fp32).  A thread's vectors of a batch are all
    // requested before any is used, so a row costs one memory round trip, not one per vector.
    float ss = 0.f;
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kNormBatch * kNormThreads) {
        uint4 yr[kNormBatch], zr[kNormBatch];
#pragma unroll
        for (int i = 0; i < kNormBatch; ++i) {
            const int v = v0 + i * kNormThreads;
            if (v < nvec) {
                yr[i] = __ldcs(y4 + v);  // read once: evict first
                zr[i] = __ldcs(z4 + v);
            }
        }
#pragma unroll
        for (int i = 0; i < kNormBatch; ++i) {
            const int v = v0 + i * kNormThreads;
            if (v < nvec) {
                const T *ye = reinterpret_cast<const T *>(&yr[i]);
                const T *ze = reinterpret_cast<const T *>(&zr[i]);
                float g[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    g[e] = to_f(ye[e]) * silu_fast(to_f(ze[e]));
                    ss = fmaf(g[e], g[e], ss);
                }
                float4 *dst = reinterpret_cast<float4 *>(g_s + v * VEC);
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q)
                    dst[q] = make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
            }
        }
    }
    // ---- CTA sum ----
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) tot += red[i];
    const float rinv = 1.f / sqrtf(tot / (float)GS + eps);

    // ---- pass 2: scale and store (each thread re-reads only what it staged) ----
    const float4 *w4 = reinterpret_cast<const float4 *>(w + (size_t)blockIdx.y * GS);
    uint4 *o4 = reinterpret_cast<uint4 *>(out + base);
    for (int v = threadIdx.x; v < nvec; v += kNormThreads) {
        const float4 *src = reinterpret_cast<const float4 *>(g_s + v * VEC);
        uint4 packed;
        T *oe = reinterpret_cast<T *>(&packed);
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
            const float4 g = src[q];
            const float4 wv = __ldg(w4 + v * (VEC / 4) + q);
            oe[4 * q + 0] = from_f<T>(g.x * rinv * wv.x);
            oe[4 * q + 1] = from_f<T>(g.y * rinv * wv.y);
            oe[4 * q + 2] = from_f<T>(g.z * rinv * wv.z);
            oe[4 * q + 3] = from_f<T>(g.w * rinv * wv.w);
        }
        __stcs(o4 + v, packed);
    }
    allow_dependents();
}

template <typename T>
static cudaError_t norm_launch(const void *y, const void *z, const float *w, void *out, int T_rows, int C,
                               int n_groups, float eps, cudaStream_t st) {
    const int GS = C / n_groups;
    const int smem = GS * (int)sizeof(float);
    if (smem > 48 * 1024) {  // once per device, to the largest group supported
        cudaError_t e = raise_smem_limit<gated_rmsnorm_kernel<T>>(kNormMaxGroup * (int)sizeof(float));
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(gated_rmsnorm_kernel<T>, dim3(T_rows, n_groups), dim3(kNormThreads), smem, st,
                      (const T *)y, (const T *)z, w, (T *)out, C, GS, eps);
}

cudaError_t launch_gated_rmsnorm(int dtype, const void *y, const void *z, const float *w, void *out, int T_rows,
                                 int C, int n_groups, float eps, cudaStream_t st) {
    if (dtype == SSD_DTYPE_BF16)
        return norm_launch<__nv_bfloat16>(y, z, w, out, T_rows, C, n_groups, eps, st);
    return norm_launch<float>(y, z, w, out, T_rows, C, n_groups, eps, st);
}

}  // namespace ssd
