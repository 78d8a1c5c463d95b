// decode_step.cu -- step a6: one cached decode step of one layer, fused into one kernel.
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
// Data movement.  The fp32 state row h[b][h][p][:] (N floats) is the only large array;
// each is read once and written once with 16-byte loads/stores, a row spread over
// N/4 consecutive lanes, so a warp moves 512 contiguous bytes per instruction.  Every
// independent load (state rows, conv windows, taps, dt) is issued before any of them is
// used, so the kernel pays about one memory round trip rather than a chain of them.
//
// Work split.  One CTA per (batch, ROWS consecutive state rows) -- always inside one head
// because P % ROWS == 0 (ROWS = 16 at small batch for parallelism, 64 otherwise so the
// shared B/C conv below is amortised over more state).  The CTA convolves its own ROWS
// x-channels (it is their only reader and writer) and all 2N B/C channels of its group,
// which every CTA of the group needs.  Those B/C conv-cache entries may only be rolled
// after every CTA of the group has read them: each CTA bumps a per-(batch, group) arrival
// counter as soon as its reads are done -- from a thread that has issued no global store, so
// its fence costs nothing and the atomic overlaps the state update -- and the CTA that arrives
// last rolls the B/C cache at its end and resets the counter to zero (no CTA ever waits, so
// nothing can hang).  The kernel has no bounded waits: it resets the workspace status word to
// SSD_OK and never sets it otherwise.
#include "common.cuh"
#include "launch.h"

namespace ssd {

// THREADS = 128 with 16 rows per CTA (small batches: more CTAs), 256 with 64 rows: 8 float4 of
// state per thread (64 registers), four CTAs to an SM.
template <typename T, int N, int K, int ROWS, int THREADS>
__global__ void __launch_bounds__(THREADS) decode_step_kernel(
    float *__restrict__ ssm, T *__restrict__ conv_state, const T *__restrict__ xBC_t,
    const T *__restrict__ dt_t, const float *__restrict__ A_log, const float *__restrict__ D,
    const float *__restrict__ dt_bias, float dt_min, float dt_max, const T *__restrict__ conv_w,
    const T *__restrict__ conv_b, T *__restrict__ y_t, int H, int P, int G, int *__restrict__ status,
    unsigned *__restrict__ counters) {
    constexpr int V = (N > 128) ? N / 128 : 1;  // float4 per thread per row
    constexpr int TPR = N / (4 * V);            // threads per row (<= 32, power of two)
    constexpr int RPP = THREADS / TPR;      // rows per pass
    constexpr int PASSES = (ROWS + RPP - 1) / RPP;
    constexpr int BC_PER = (2 * N + THREADS - 1) / THREADS;  // B/C channels per thread

    __shared__ float uB[N], uC[N], ux[ROWS];
    __shared__ float s_dt, s_a, s_d;
    __shared__ int s_last;

    const int b = blockIdx.y;
    const int row0 = blockIdx.x * ROWS;  // first (h*P + p) row of this CTA
    const int h = row0 / P;
    const int g = h / (H / G);
    const int HP = H * P, GN = G * N;
    const int Cc = HP + 2 * GN;
    const int tid = threadIdx.x;
    const int r_in_pass = tid / TPR, lane_in_row = tid % TPR;
    constexpr int kArriver = THREADS - 1;  // no x channel (ROWS < THREADS): no store before the arrival
    static_assert(ROWS < THREADS, "the arriving thread must not own an x channel");

    grid_dependency_wait();  // every global access comes after the kernel before
    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *status = SSD_OK;

    // ---- issue every independent load first ----
    float4 st[PASSES][V];
    float *ssm_b = ssm + ((size_t)b * HP + row0) * N;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
        const int r = ps * RPP + r_in_pass;
#pragma unroll
        for (int v = 0; v < V; ++v)
            if (r < ROWS)
                st[ps][v] = *reinterpret_cast<const float4 *>(ssm_b + (size_t)r * N + (v * TPR + lane_in_row) * 4);
    }
    // B/C channels of group g (read-only here)
    float bc_win[BC_PER][K], bc_w[BC_PER][K], bc_bias[BC_PER];
#pragma unroll
    for (int q = 0; q < BC_PER; ++q) {
        const int i = tid + q * THREADS;
        if (i < 2 * N) {
            const int cc = HP + (i < N ? g * N + i : GN + g * N + (i - N));
            const T *cs = conv_state + ((size_t)b * Cc + cc) * (K - 1);
#pragma unroll
            for (int k = 0; k < K - 1; ++k) bc_win[q][k] = to_f(cs[k]);
            bc_win[q][K - 1] = to_f(__ldg(xBC_t + (size_t)b * Cc + cc));
#pragma unroll
            for (int k = 0; k < K; ++k) bc_w[q][k] = to_f(__ldg(conv_w + (size_t)cc * K + k));
            bc_bias[q] = conv_b ? to_f(__ldg(conv_b + cc)) : 0.f;
        }
    }
    // this CTA's own x channels
    T x_win[K];
    float x_w[K], x_bias = 0.f;
    if (tid < ROWS) {
        const int cc = row0 + tid;
        const T *cs = conv_state + ((size_t)b * Cc + cc) * (K - 1);
#pragma unroll
        for (int k = 0; k < K - 1; ++k) x_win[k] = cs[k];
        x_win[K - 1] = __ldg(xBC_t + (size_t)b * Cc + cc);
#pragma unroll
        for (int k = 0; k < K; ++k) x_w[k] = to_f(__ldg(conv_w + (size_t)cc * K + k));
        x_bias = conv_b ? to_f(__ldg(conv_b + cc)) : 0.f;
    }
    float dt_raw = 0.f, alog = 0.f, dbias = 0.f, dskip = 0.f;
    if (tid == 0) {
        dt_raw = to_f(__ldg(dt_t + (size_t)b * H + h));
        alog = __ldg(A_log + h);
        dbias = dt_bias ? __ldg(dt_bias + h) : 0.f;
        dskip = D ? __ldg(D + h) : 0.f;
    }

    // ---- conv outputs, x-channel cache roll, discretisation ----
#pragma unroll
    for (int q = 0; q < BC_PER; ++q) {
        const int i = tid + q * THREADS;
        if (i < 2 * N) {
            float acc = bc_bias[q];
#pragma unroll
            for (int k = 0; k < K; ++k) acc = fmaf(bc_w[q][k], bc_win[q][k], acc);
            const float u = silu_f(acc);
            if (i < N) uB[i] = u; else uC[i - N] = u;
        }
    }
    if (tid < ROWS) {
        float acc = x_bias;
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(x_w[k], to_f(x_win[k]), acc);
        ux[tid] = silu_f(acc);
        T *cs = conv_state + ((size_t)b * Cc + row0 + tid) * (K - 1);
#pragma unroll
        for (int k = 0; k < K - 1; ++k) cs[k] = x_win[k + 1];
    }
    if (tid == 0) {
        const float dt = discretise_dt(dt_raw, dbias, dt_min, dt_max);
        s_dt = dt;
        s_a = expf(dt * -expf(alog));
        s_d = dskip;
    }
    __syncthreads();  // conv outputs and dt are in shared memory; B/C cache reads are done

    // ---- arrival: the CTA that arrives last for its (batch, group) rolls the B/C cache below ----
    if (tid == kArriver) {
        __threadfence();
        const unsigned ctas = (unsigned)((H / G) * P / ROWS);
        const unsigned prev = atomicAdd(&counters[b * G + g], 1u);
        s_last = (prev == ctas - 1);
    }

    // ---- state update and output ----
    const float dt = s_dt, a = s_a, dsk = s_d;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
        const int r = ps * RPP + r_in_pass;
        float part = 0.f;
        float xv = 0.f;
        if (r < ROWS) {
            xv = ux[r];
            const float dx = dt * xv;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int n = (v * TPR + lane_in_row) * 4;
                float4 s = st[ps][v];
                s.x = fmaf(a, s.x, dx * uB[n + 0]);
                s.y = fmaf(a, s.y, dx * uB[n + 1]);
                s.z = fmaf(a, s.z, dx * uB[n + 2]);
                s.w = fmaf(a, s.w, dx * uB[n + 3]);
                part = fmaf(s.x, uC[n + 0], part);
                part = fmaf(s.y, uC[n + 1], part);
                part = fmaf(s.z, uC[n + 2], part);
                part = fmaf(s.w, uC[n + 3], part);
                *reinterpret_cast<float4 *>(ssm_b + (size_t)r * N + n) = s;
            }
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o, TPR);
        if (r < ROWS && lane_in_row == 0) y_t[(size_t)b * HP + row0 + r] = from_f<T>(part + dsk * xv);
    }

    __syncthreads();  // s_last is visible
    if (s_last) {
        // every CTA of this (batch, group) has read the B/C cache: roll it
        __threadfence();
#pragma unroll
        for (int q = 0; q < BC_PER; ++q) {
            const int i = tid + q * THREADS;
            if (i < 2 * N) {
                const int cc = HP + (i < N ? g * N + i : GN + g * N + (i - N));
                T *cs = conv_state + ((size_t)b * Cc + cc) * (K - 1);
#pragma unroll
                for (int k = 0; k < K - 1; ++k) cs[k] = from_f<T>(bc_win[q][k + 1]);
            }
        }
        if (tid == 0) atomicExch(&counters[b * G + g], 0u);
    }
    allow_dependents();
}

template <typename T, int N, int K, int ROWS, int THREADS>
static cudaError_t decode_launch(float *ssm, void *conv_state, const void *xBC_t, const void *dt_t,
                                 const float *A_log, const float *D, const float *dt_bias, float dt_min,
                                 float dt_max, const void *conv_w, const void *conv_b, void *y_t,
                                 int B, int H, int P, int G, int *status, unsigned *counters, cudaStream_t st) {
    dim3 grid(H * P / ROWS, B);
    return launch_pdl(decode_step_kernel<T, N, K, ROWS, THREADS>, grid, dim3(THREADS), 0, st, ssm, (T *)conv_state,
                      (const T *)xBC_t, (const T *)dt_t, A_log, D, dt_bias, dt_min, dt_max, (const T *)conv_w,
                      (const T *)conv_b, (T *)y_t, H, P, G, status, counters);
}

template <typename T, int N, int K>
static cudaError_t decode_rows(bool wide, float *ssm, void *conv_state, const void *xBC_t, const void *dt_t,
                               const float *A_log, const float *D, const float *dt_bias, float dt_min,
                               float dt_max, const void *conv_w, const void *conv_b, void *y_t, int B,
                               int H, int P, int G, int *status, unsigned *counters, cudaStream_t st) {
    if (wide)
        return decode_launch<T, N, K, 64, 256>(ssm, conv_state, xBC_t, dt_t, A_log, D, dt_bias, dt_min, dt_max,
                                          conv_w, conv_b, y_t, B, H, P, G, status, counters, st);
    return decode_launch<T, N, K, 16, 128>(ssm, conv_state, xBC_t, dt_t, A_log, D, dt_bias, dt_min, dt_max,
                                      conv_w, conv_b, y_t, B, H, P, G, status, counters, st);
}

template <typename T, int N>
static cudaError_t decode_k(int K, bool wide, float *ssm, void *conv_state, const void *xBC_t,
                            const void *dt_t, const float *A_log, const float *D, const float *dt_bias,
                            float dt_min, float dt_max, const void *conv_w, const void *conv_b, void *y_t,
                            int B, int H, int P, int G, int *status, unsigned *counters, cudaStream_t st) {
#define SSD_DK(KK)                                                                                   \
    case KK:                                                                                         \
        return decode_rows<T, N, KK>(wide, ssm, conv_state, xBC_t, dt_t, A_log, D, dt_bias, dt_min, \
                                     dt_max, conv_w, conv_b, y_t, B, H, P, G, status, counters, st);
    switch (K) {
        SSD_DK(2) SSD_DK(3) SSD_DK(4) SSD_DK(5) SSD_DK(6) SSD_DK(7) SSD_DK(8)
    }
#undef SSD_DK
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_step(int dtype, float *ssm_state, void *conv_state, const void *xBC_t,
                               const void *dt_t, const float *A_log, const float *D,
                               const float *dt_bias, float dt_min, float dt_max,
                               const void *conv_w, const void *conv_b, void *y_t, int B, int H,
                               int P, int G, int N, int K, int *status, unsigned *counters,
                               cudaStream_t st) {
    // 64 rows per CTA once the batch gives enough CTAs; 16 otherwise
    const bool wide = (P % 64 == 0) && (B >= 4);
#define SSD_DN(T, NN)                                                                              \
    case NN:                                                                                       \
        return decode_k<T, NN>(K, wide, ssm_state, conv_state, xBC_t, dt_t, A_log, D, dt_bias,      \
                               dt_min, dt_max, conv_w, conv_b, y_t, B, H, P, G, status, counters, st);
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
