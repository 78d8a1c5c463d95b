// decode_step.cu -- step a6: one cached decode step of one layer, as two kernels.
//
//   window = [conv_state[c][0..K-2], xBC_t[c]]                      (oldest .. newest)
//   u[c]   = SiLU(sum_k w[c][k] window[k] + b[c]);  conv_state[c] <- window[1..K-1]
//   x | B | C = u split by channel;  dt = clip(softplus(dt_t + dt_bias))
//   h <- exp(dt * -exp(A_log)) h + dt x (outer) B;   y = h C + D x
//
// Source: blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §2.1 (constant-size state, conv cache
// of kernel_size-1 inputs), §2.2 (Mamba2Cache.update: roll the conv window, set the
// newest slot, ssm = ssm * A_bar + B_bar * x), §3.2 (decode is bandwidth bound; the
// state update runs in float32).
//
// Split.  The fp32 state h[b][h][p][:] is the only large array (B*H*P*N*4 bytes read and
// written); everything else is a few bytes per channel.  The step runs as
//   1. decode_conv_kernel: one thread per (batch, channel) convolves the window, writes
//      u = SiLU(conv) to the workspace as fp32 and rolls conv_state in place; threads of the
//      first CTA of each batch also write (dt, exp(dt*A)) per head.  Every channel has exactly
//      one reader and one writer here, so the roll needs no cross-CTA protocol.
//   2. decode_state_kernel: one CTA per (batch, ROWS consecutive state rows), barrier-free.
//      Each thread streams its share of the rows with 16-byte loads and stores (a row over
//      N/4 consecutive lanes, 512 contiguous bytes per warp instruction) and takes its x, B,
//      C and (dt, a) from the workspace, where kernel 1 has just left them in L2.
//
// Overlap.  Both kernels are launched with programmatic dependent launch.  Kernel 1 allows
// its dependents as soon as its own dependency wait returns, i.e. once every kernel before
// this step has completed.  Kernel 2 is therefore only ever scheduled after that point, and
// kernel 1 never touches the state, so kernel 2 issues its state loads BEFORE its own
// dependency wait: the state's DRAM latency overlaps kernel 1.  Those loads go through L2
// only (ld.global.cg), the level at which the completed earlier kernels' stores are
// performed, so no SM's L1 can serve a stale line.  Everything kernel 1 wrote is read after
// the wait.  Neither kernel waits on anything else: there are no spin-waits and no bounded
// waits; kernel 2 resets the workspace status word to SSD_OK and never sets it otherwise.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace ssd {

constexpr int kConvThreads = 256;

// Loads and stores of one bf16 or fp32 element with an L2 eviction-priority policy: the conv
// kernel keeps the conv windows and taps evict_last, so that the 64-layer stream of states
// between two steps of a layer does not push them out of L2.
template <typename T> __device__ __forceinline__ T ld_policy(const T *p, uint64_t pol);
template <> __device__ __forceinline__ __nv_bfloat16 ld_policy(const __nv_bfloat16 *p, uint64_t pol) {
    unsigned short v;
    asm volatile("ld.global.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(v) : "l"(p), "l"(pol));
    return __ushort_as_bfloat16(v);
}
template <> __device__ __forceinline__ float ld_policy(const float *p, uint64_t pol) {
    float v;
    asm volatile("ld.global.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(p), "l"(pol));
    return v;
}
template <typename T> __device__ __forceinline__ void st_policy(T *p, T v, uint64_t pol);
template <> __device__ __forceinline__ void st_policy(__nv_bfloat16 *p, __nv_bfloat16 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(__bfloat16_as_ushort(v)), "l"(pol)
                 : "memory");
}
template <> __device__ __forceinline__ void st_policy(float *p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads) decode_conv_kernel(
    T *__restrict__ conv_state, const T *__restrict__ xBC_t, const T *__restrict__ dt_t,
    const float *__restrict__ A_log, const float *__restrict__ dt_bias, float dt_min, float dt_max,
    const T *__restrict__ conv_w, const T *__restrict__ conv_b, float *__restrict__ u_ws,
    float2 *__restrict__ da_ws, int H, int Cc) {
    grid_dependency_wait();  // every global access comes after the kernels before this step
    allow_dependents();      // the state kernel may start streaming the state now
    conv_state = after_wait(conv_state);
    xBC_t = after_wait(xBC_t);
    dt_t = after_wait(dt_t);
    A_log = after_wait(A_log);
    dt_bias = after_wait(dt_bias);
    conv_w = after_wait(conv_w);
    conv_b = after_wait(conv_b);
    u_ws = after_wait(u_ws);
    da_ws = after_wait(da_ws);
    const int b = blockIdx.y;
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    if (c < Cc) {
        const uint64_t keep = tc::l2_evict_last();
        T *cs = conv_state + ((size_t)b * Cc + c) * (K - 1);
        T win[K];
        float w[K];
#pragma unroll
        for (int k = 0; k < K - 1; ++k) win[k] = ld_policy(cs + k, keep);
        win[K - 1] = __ldg(xBC_t + (size_t)b * Cc + c);
#pragma unroll
        for (int k = 0; k < K; ++k) w[k] = to_f(ld_policy(conv_w + (size_t)c * K + k, keep));
        float acc = conv_b ? to_f(ld_policy(conv_b + c, keep)) : 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(w[k], to_f(win[k]), acc);
        u_ws[(size_t)b * Cc + c] = silu_f(acc);
#pragma unroll
        for (int k = 0; k < K - 1; ++k) st_policy(cs + k, win[k + 1], keep);
    }
    if (blockIdx.x == 0)
        for (int h = threadIdx.x; h < H; h += kConvThreads) {
            const float raw = to_f(__ldg(dt_t + (size_t)b * H + h));
            const float dt = discretise_dt(raw, dt_bias ? __ldg(dt_bias + h) : 0.f, dt_min, dt_max);
            da_ws[(size_t)b * H + h] = make_float2(dt, expf(dt * -expf(__ldg(A_log + h))));
        }
}

// ROWS = 16 state rows per CTA, always inside one head because P % 16 == 0.  A row is N/4
// float4 spread over TPR lanes (V float4 each, V = 2 only for N = 256); a 128-thread CTA
// covers RPP rows per pass.  16-row CTAs measured fastest at batch 1 and batch 16 alike:
// small CTAs with no barrier keep the most state bytes in flight per SM.
template <typename T, int N, int ROWS, int THREADS>
__global__ void __launch_bounds__(THREADS) decode_state_kernel(
    float *__restrict__ ssm, const float *__restrict__ u_ws, const float2 *__restrict__ da_ws,
    const float *__restrict__ D, T *__restrict__ y_t, int H, int P, int G, int *__restrict__ status,
    int stream_first) {
    constexpr int V = (N > 128) ? N / 128 : 1;  // float4 per thread per row
    constexpr int TPR = N / (4 * V);            // threads per row (<= 32, power of two)
    constexpr int RPP = THREADS / TPR;          // rows per pass
    constexpr int PASSES = (ROWS + RPP - 1) / RPP;
    static_assert(THREADS % TPR == 0 && TPR <= 32, "a row's lanes must sit in one warp");

    const int b = blockIdx.y;
    const int row0 = blockIdx.x * ROWS;  // first (h*P + p) row of this CTA
    const int h = row0 / P;
    const int g = h / (H / G);
    const int HP = H * P, GN = G * N;
    const int Cc = HP + 2 * GN;
    const int r_in_pass = threadIdx.x / TPR, lane_in_row = threadIdx.x % TPR;

    // ---- the state, before the dependency wait: L2-only loads (see the file comment) ----
    // With stream_first the state's lines are loaded and stored evict_first: at small batches
    // that keeps the step's small data (the conv windows and taps, the conv outputs) in L2
    // across the 64-layer stream of states.
    const uint64_t first_policy = tc::l2_evict_first();
    float4 st[PASSES][V];
    float *ssm_b = ssm + ((size_t)b * HP + row0) * N;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
        const int r = ps * RPP + r_in_pass;
#pragma unroll
        for (int v = 0; v < V; ++v)
            if (r < ROWS)
            {
                const float4 *src = reinterpret_cast<const float4 *>(ssm_b + (size_t)r * N + (v * TPR + lane_in_row) * 4);
                st[ps][v] = stream_first ? ldcg_hint(src, first_policy) : __ldcg(src);
            }
    }

    grid_dependency_wait();  // the conv kernel's u and (dt, a) are complete and visible
    u_ws = after_wait(u_ws);
    da_ws = after_wait(da_ws);
    D = after_wait(D);
    y_t = after_wait(y_t);
    status = after_wait(status);
    ssm_b = after_wait(ssm_b);  // the stores (the loads above are the deliberate early reads)
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status = SSD_OK;

    // ---- x, B, C and (dt, a) of this step, from the workspace ----
    const float *u_b = u_ws + (size_t)b * Cc;
    float4 uB[V], uC[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int n = (v * TPR + lane_in_row) * 4;
        uB[v] = *reinterpret_cast<const float4 *>(u_b + HP + g * N + n);
        uC[v] = *reinterpret_cast<const float4 *>(u_b + HP + GN + g * N + n);
    }
    float xs[PASSES];
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
        const int r = ps * RPP + r_in_pass;
        xs[ps] = r < ROWS ? u_b[row0 + r] : 0.f;
    }
    const float2 da = da_ws[(size_t)b * H + h];
    const float dsk = D ? __ldg(D + h) : 0.f;

    // ---- state update and output ----
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
        const int r = ps * RPP + r_in_pass;
        const float xv = xs[ps];
        float part = 0.f;
        if (r < ROWS) {
            const float dx = da.x * xv;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float4 s = st[ps][v];
                s.x = fmaf(da.y, s.x, dx * uB[v].x);
                s.y = fmaf(da.y, s.y, dx * uB[v].y);
                s.z = fmaf(da.y, s.z, dx * uB[v].z);
                s.w = fmaf(da.y, s.w, dx * uB[v].w);
                part = fmaf(s.x, uC[v].x, part);
                part = fmaf(s.y, uC[v].y, part);
                part = fmaf(s.z, uC[v].z, part);
                part = fmaf(s.w, uC[v].w, part);
                float4 *dst = reinterpret_cast<float4 *>(ssm_b + (size_t)r * N + (v * TPR + lane_in_row) * 4);
                if (stream_first)
                    st_global_hint_v4(dst, s, first_policy);
                else
                    *dst = s;
            }
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o, TPR);
        if (r < ROWS && lane_in_row == 0) y_t[(size_t)b * HP + row0 + r] = from_f<T>(part + dsk * xv);
    }
    allow_dependents();
}

template <typename T>
static cudaError_t conv_k(int K, void *conv_state, const void *xBC_t, const void *dt_t, const float *A_log,
                          const float *dt_bias, float dt_min, float dt_max, const void *conv_w,
                          const void *conv_b, float *u_ws, float2 *da_ws, int B, int H, int Cc,
                          cudaStream_t st) {
    const dim3 grid(cdiv(Cc, kConvThreads), B);
#define SSD_CK(KK)                                                                                   \
    case KK:                                                                                         \
        return launch_pdl(decode_conv_kernel<T, KK>, grid, dim3(kConvThreads), 0, st, (T *)conv_state, \
                          (const T *)xBC_t, (const T *)dt_t, A_log, dt_bias, dt_min, dt_max,        \
                          (const T *)conv_w, (const T *)conv_b, u_ws, da_ws, H, Cc);
    switch (K) {
        SSD_CK(2) SSD_CK(3) SSD_CK(4) SSD_CK(5) SSD_CK(6) SSD_CK(7) SSD_CK(8)
    }
#undef SSD_CK
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_conv(int dtype, void *conv_state, const void *xBC_t, const void *dt_t,
                               const float *A_log, const float *dt_bias, float dt_min, float dt_max,
                               const void *conv_w, const void *conv_b, float *u_ws, float2 *da_ws,
                               int B, int H, int P, int G, int N, int K, cudaStream_t st) {
    const int Cc = H * P + 2 * G * N;
    if (dtype == SSD_DTYPE_BF16)
        return conv_k<__nv_bfloat16>(K, conv_state, xBC_t, dt_t, A_log, dt_bias, dt_min, dt_max, conv_w,
                                     conv_b, u_ws, da_ws, B, H, Cc, st);
    return conv_k<float>(K, conv_state, xBC_t, dt_t, A_log, dt_bias, dt_min, dt_max, conv_w, conv_b, u_ws,
                         da_ws, B, H, Cc, st);
}

// Batches up to this size stream the state evict_first.  Measured on the 64-layer 2.7B-shaped
// decode (steps/s, against the default policy): +14 % at batch 1, +5 % at 2, +1 % at 4, -3 % at
// 8 and 16.
constexpr int kStreamFirstMaxB = 4;

template <typename T, int N>
static cudaError_t state_launch(float *ssm, const float *u_ws, const float2 *da_ws, const float *D, void *y_t,
                                int B, int H, int P, int G, int *status, cudaStream_t st) {
    constexpr int ROWS = 16;
    constexpr int TPR = N / (4 * ((N > 128) ? N / 128 : 1));
    constexpr int THREADS = ROWS * TPR < 128 ? ROWS * TPR : 128;
    const dim3 grid(H * P / ROWS, B);
    return launch_pdl(decode_state_kernel<T, N, ROWS, THREADS>, grid, dim3(THREADS), 0, st, ssm, u_ws, da_ws,
                      D, (T *)y_t, H, P, G, status, B <= kStreamFirstMaxB ? 1 : 0);
}

cudaError_t launch_decode_state(int dtype, float *ssm_state, const float *u_ws, const float2 *da_ws,
                                const float *D, void *y_t, int B, int H, int P, int G, int N, int *status,
                                cudaStream_t st) {
#define SSD_DN(T, NN) \
    case NN:          \
        return state_launch<T, NN>(ssm_state, u_ws, da_ws, D, y_t, B, H, P, G, status, st);
    if (dtype == SSD_DTYPE_BF16) {
        switch (N) { SSD_DN(__nv_bfloat16, 16) SSD_DN(__nv_bfloat16, 32) SSD_DN(__nv_bfloat16, 64)
                     SSD_DN(__nv_bfloat16, 128) SSD_DN(__nv_bfloat16, 256) }
    } else {
        switch (N) { SSD_DN(float, 16) SSD_DN(float, 32) SSD_DN(float, 64) SSD_DN(float, 128)
                     SSD_DN(float, 256) }
    }
#undef SSD_DN
    return cudaErrorInvalidValue;
}

}  // namespace ssd
