// causal_conv1d.cu -- support step a7: depthwise causal conv1d + bias + SiLU over a
// prefix, and the conv cache (the last K-1 raw inputs, oldest first) that cached decode
// continues from.
//
//   out[b][t][c] = SiLU(sum_k w[c][k] xBC[b][t-K+1+k][c] + bias[c]),  zero left padding
//
// Source: blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §2.1: a fixed-size (kernel_size - 1)
// input cache for the depthwise conv, kept beside the SSM state.
//
// One thread per (group of 4 channels, 32-token strip): 4 bf16 channels as one 8-byte vector,
// or 4 fp32 channels as one 16-byte vector, so a warp moves 256 (bf16) or 512 (fp32)
// contiguous bytes per instruction.  The thread keeps the K-1 previous inputs of its channels in registers and
// slides along the strip, requesting 8 tokens' vectors at once before using any of them, so a
// strip costs a few memory round trips rather than one per token.  Each input is read once,
// plus K-1 halo tokens per strip (about 9 %, mostly from L2).  Launched with programmatic
// dependent launch: xBC comes from the kernel before.
#include "common.cuh"
#include "launch.h"

namespace ssd {

constexpr int kStrip = 32;       // tokens per thread
constexpr int kConvBatch = 8;    // tokens requested together
constexpr int kConvThreads = 128;
constexpr int kConvCh = 4;       // channels per thread: 8-byte bf16 or 16-byte fp32 vectors

template <typename T>
struct ConvVec {
    using type = uint2;  // 4 bf16
};
template <>
struct ConvVec<float> {
    using type = uint4;  // 4 fp32
};

template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads) causal_conv1d_kernel(
    const T *__restrict__ xBC, const T *__restrict__ w, const T *__restrict__ bias,
    T *__restrict__ out, T *__restrict__ conv_state_out, int L, int Cc) {
    constexpr int VEC = kConvCh;  // channels per thread
    using VT = typename ConvVec<T>::type;
    grid_dependency_wait();
    xBC = after_wait(xBC);
    w = after_wait(w);
    bias = after_wait(bias);
    out = after_wait(out);
    conv_state_out = after_wait(conv_state_out);

    const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * VEC;
    const int t0 = blockIdx.y * kStrip;
    const int b = blockIdx.z;
    if (c0 < Cc) {
        // taps [VEC][K] and bias, as 16-byte vectors (c0 * K * sizeof(T) is a multiple of 16)
        float wk[VEC][K], bc[VEC];
        {
            const VT *w4 = reinterpret_cast<const VT *>(w + (size_t)c0 * K);
#pragma unroll
            for (int i = 0; i < K; ++i) {
                const VT r = __ldg(w4 + i);
                const T *e = reinterpret_cast<const T *>(&r);
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    const int f = i * VEC + j;  // flat index into [VEC][K]
                    wk[f / K][f % K] = to_f(e[j]);
                }
            }
            if (bias) {
                const VT r = __ldg(reinterpret_cast<const VT *>(bias + c0));
                const T *e = reinterpret_cast<const T *>(&r);
#pragma unroll
                for (int j = 0; j < VEC; ++j) bc[j] = to_f(e[j]);
            } else {
#pragma unroll
                for (int j = 0; j < VEC; ++j) bc[j] = 0.f;
            }
        }
        const T *xb = xBC + (size_t)b * L * Cc + c0;
        T *ob = out + (size_t)b * L * Cc + c0;
        // the window: win[k] holds token t - (K-1) + k for the next output t
        float win[K - 1][VEC];
#pragma unroll
        for (int k = 0; k < K - 1; ++k) {
            const int s = t0 - (K - 1) + k;
            VT r = {};
            if (s >= 0) r = *reinterpret_cast<const VT *>(xb + (size_t)s * Cc);
            const T *e = reinterpret_cast<const T *>(&r);
#pragma unroll
            for (int j = 0; j < VEC; ++j) win[k][j] = s >= 0 ? to_f(e[j]) : 0.f;
        }
        const int t1 = min(L, t0 + kStrip);
        for (int tb = t0; tb < t1; tb += kConvBatch) {
            VT r[kConvBatch];
#pragma unroll
            for (int i = 0; i < kConvBatch; ++i)
                if (tb + i < t1) r[i] = __ldcs(reinterpret_cast<const VT *>(xb + (size_t)(tb + i) * Cc));
#pragma unroll
            for (int i = 0; i < kConvBatch; ++i) {
                if (tb + i < t1) {
                    const T *e = reinterpret_cast<const T *>(&r[i]);
                    VT o;
                    T *oe = reinterpret_cast<T *>(&o);
#pragma unroll
                    for (int j = 0; j < VEC; ++j) {
                        const float newest = to_f(e[j]);
                        float acc = bc[j];
#pragma unroll
                        for (int k = 0; k < K - 1; ++k) acc = fmaf(wk[j][k], win[k][j], acc);
                        acc = fmaf(wk[j][K - 1], newest, acc);
                        oe[j] = from_f<T>(silu_fast(acc));
#pragma unroll
                        for (int k = 0; k < K - 2; ++k) win[k][j] = win[k + 1][j];
                        win[K - 2][j] = newest;
                    }
                    __stcs(reinterpret_cast<VT *>(ob + (size_t)(tb + i) * Cc), o);
                }
            }
        }
        // the conv cache: the last K-1 raw inputs of the sequence, oldest first, 0 before the start
        if (conv_state_out && blockIdx.y == 0) {
            for (int j = 0; j < K - 1; ++j) {
                const int s = L - (K - 1) + j;
                VT r = {};
                if (s >= 0) r = *reinterpret_cast<const VT *>(xb + (size_t)s * Cc);
                const T *e = reinterpret_cast<const T *>(&r);
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    conv_state_out[((size_t)b * Cc + c0 + v) * (K - 1) + j] = s >= 0 ? e[v] : from_f<T>(0.f);
            }
        }
    }
    allow_dependents();
}

template <typename T>
static cudaError_t conv_launch(const void *xBC, const void *conv_w, const void *conv_b, void *out,
                               void *conv_state_out, int B, int L, int Cc, int K, cudaStream_t st) {
    constexpr int VEC = kConvCh;
    const dim3 grid(cdiv(Cc / VEC, kConvThreads), cdiv(L > 0 ? L : 1, kStrip), B);
#define SSD_CV(KK)                                                                                       \
    case KK:                                                                                             \
        return launch_pdl(causal_conv1d_kernel<T, KK>, grid, dim3(kConvThreads), 0, st, (const T *)xBC,  \
                          (const T *)conv_w, (const T *)conv_b, (T *)out, (T *)conv_state_out, L, Cc);
    switch (K) {
        SSD_CV(2) SSD_CV(3) SSD_CV(4) SSD_CV(5) SSD_CV(6) SSD_CV(7) SSD_CV(8)
    }
#undef SSD_CV
    return cudaErrorInvalidValue;
}

cudaError_t launch_causal_conv1d(int dtype, const void *xBC, const void *conv_w,
                                 const void *conv_b, void *out, void *conv_state_out, int B,
                                 int L, int Cc, int K, cudaStream_t st) {
    if (dtype == SSD_DTYPE_BF16)
        return conv_launch<__nv_bfloat16>(xBC, conv_w, conv_b, out, conv_state_out, B, L, Cc, K, st);
    return conv_launch<float>(xBC, conv_w, conv_b, out, conv_state_out, B, L, Cc, K, st);
}

}  // namespace ssd
