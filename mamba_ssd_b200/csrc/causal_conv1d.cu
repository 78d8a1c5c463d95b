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
// One thread per (channel, 64-token strip): the thread keeps its K-1 previous inputs in
// registers and slides along the strip, so each input is read once (plus K-1 halo
// reads per strip); consecutive threads read consecutive channels (coalesced rows).
#include "common.cuh"
#include "launch.h"

namespace ssd {

constexpr int kStrip = 64;
constexpr int kConvMaxK = 8;

template <typename T>
__global__ void __launch_bounds__(128) causal_conv1d_kernel(
    const T *__restrict__ xBC, const T *__restrict__ w, const T *__restrict__ bias,
    T *__restrict__ out, T *__restrict__ conv_state_out, int L, int Cc, int K) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int t0 = blockIdx.y * kStrip;
    const int b = blockIdx.z;
    if (c >= Cc) return;
    float wk[kConvMaxK];
    for (int k = 0; k < K; ++k) wk[k] = to_f(w[(size_t)c * K + k]);
    const float bc = bias ? to_f(bias[c]) : 0.f;
    const T *xb = xBC + (size_t)b * L * Cc + c;
    float win[kConvMaxK];  // win[K-1] is the newest
    for (int k = 0; k < K - 1; ++k) {
        const int s = t0 - (K - 1) + k;
        win[k] = s >= 0 ? to_f(xb[(size_t)s * Cc]) : 0.f;
    }
    const int t1 = min(L, t0 + kStrip);
    for (int t = t0; t < t1; ++t) {
        win[K - 1] = to_f(xb[(size_t)t * Cc]);
        float acc = bc;
        for (int k = 0; k < K; ++k) acc = fmaf(wk[k], win[k], acc);
        out[((size_t)b * L + t) * Cc + c] = from_f<T>(silu_f(acc));
        for (int k = 0; k < K - 1; ++k) win[k] = win[k + 1];
    }
    if (conv_state_out && blockIdx.y == 0) {
        for (int j = 0; j < K - 1; ++j) {
            const int s = L - (K - 1) + j;
            conv_state_out[((size_t)b * Cc + c) * (K - 1) + j] =
                s >= 0 ? xb[(size_t)s * Cc] : from_f<T>(0.f);
        }
    }
}

cudaError_t launch_causal_conv1d(int dtype, const void *xBC, const void *conv_w,
                                 const void *conv_b, void *out, void *conv_state_out, int B,
                                 int L, int Cc, int K, cudaStream_t st) {
    dim3 grid(cdiv(Cc, 128), cdiv(L > 0 ? L : 1, kStrip), B);
    if (dtype == SSD_DTYPE_BF16) {
        causal_conv1d_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
            (const __nv_bfloat16 *)xBC, (const __nv_bfloat16 *)conv_w,
            (const __nv_bfloat16 *)conv_b, (__nv_bfloat16 *)out, (__nv_bfloat16 *)conv_state_out, L,
            Cc, K);
    } else {
        causal_conv1d_kernel<float><<<grid, 128, 0, st>>>((const float *)xBC, (const float *)conv_w,
                                                          (const float *)conv_b, (float *)out,
                                                          (float *)conv_state_out, L, Cc, K);
    }
    return cudaGetLastError();
}

}  // namespace ssd
