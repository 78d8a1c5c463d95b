// decay_prep.cu -- step a1 of the chunked SSD: discretisation and the per-chunk
// cumulative decay.
//
//   dt_t  = clip(softplus(dt_raw + dt_bias[h]), dt_min, dt_max)
//   dA_t  = dt_t * (-exp(A_log[h]))                        (float32, "the decay in fp32")
//   acs_t = sum of dA over the chunk up to and including t  (segsum building block)
//
// Source: "Compiler-First State Space Duality ..." blog walk-through (bqwf.cn) §1.1
// (discretisation, chunks of 256 tokens, L = tril(exp(segsum))), §1.2 (the fused
// softplus -> clip -> exp chain) and §4.1 (the decay must be float32).  The printed
// exp(softplus(A_log) * dt) has lost its sign; A = -exp(A_log) is the Mamba-2 form
// that the paper's checkpoint parity implies.
//
// One CTA per (chunk, batch, block of 8 heads): the chunk's dt values for 8 heads are
// read row by row (all loads of a thread issued together), transposed through shared
// memory, and each of the 8 warps scans one head's chunk with shuffles.  Tokens past L get dt = 0, so
// their decay is 1 and the chunk's last cumsum is that of the last real token.
#include "common.cuh"
#include "launch.h"

namespace ssd {

// Used by the CUDA-core path; the tensor-core path forms the same factors (in log2 form)
// inside its block-state kernel.
template <typename T>
__global__ void __launch_bounds__(256) decay_prep_kernel(
    const T *__restrict__ dt, const float *__restrict__ A_log, const float *__restrict__ dt_bias,
    float dt_min, float dt_max, float *__restrict__ dtf, float *__restrict__ acs,
    int *__restrict__ status, int L, int H, int Q, int nc) {
    extern __shared__ float sm[];  // [8][Q + 1]
    const int c = blockIdx.x, b = blockIdx.y, hb = blockIdx.z * 8;
    // this call's status word starts clean (later kernels of the call may set a timeout)
    if (status && c == 0 && b == 0 && blockIdx.z == 0 && threadIdx.x == 0) *status = SSD_OK;
    const int nh = min(8, H - hb);
    const int ld = Q + 1;
    // Q * 8 slots over 256 threads: at most 16 per thread (Q <= 512), loads issued together
    constexpr int kPer = 16;
    float raw[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int idx = threadIdx.x + i * 256;
        const int t = idx >> 3, j = idx & 7;
        const int tok = c * Q + t;
        raw[i] = (t < Q && j < nh && tok < L) ? to_f(dt[((size_t)b * L + tok) * H + hb + j]) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int idx = threadIdx.x + i * 256;
        const int t = idx >> 3, j = idx & 7;
        if (t < Q && j < nh) {
            const int tok = c * Q + t;
            float v = 0.f;
            if (tok < L) v = discretise_dt(raw[i], dt_bias ? dt_bias[hb + j] : 0.f, dt_min, dt_max);
            sm[j * ld + t] = v;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = Q / 32;  // tokens per lane (Q is a multiple of 32)
    const size_t Lp = (size_t)nc * Q;
    for (int j = warp; j < nh; j += 8) {  // one head per warp
        const int h = hb + j;
        const float A = -expf(A_log[h]);
        const float *row = sm + j * ld + lane * per;
        float run = 0.f;
        for (int i = 0; i < per; ++i) run += row[i] * A;
        float acc = warp_inclusive_sum(run) - run;  // exclusive prefix of this lane
        const size_t base = ((size_t)b * H + h) * Lp + (size_t)c * Q + lane * per;
        // In a ragged last chunk the padded slots must hold exactly the cumsum of the last real
        // token, the value the chunk's end stands for: the lanes' partial sums round
        // differently, and exp(acs_end - acs_last) must be exactly 1, not exp(rounding) (which
        // is far from 1, or infinite, when the cumsum is large).
        const int tl = L - 1 - c * Q;  // slot of the last real token, when the chunk is ragged
        const bool ragged = tl < Q - 1;
        float last = 0.f;
        for (int i = 0; i < per; ++i) {
            acc += row[i] * A;
            if (lane * per + i == tl) last = acc;
            acs[base + i] = acc;
            dtf[base + i] = row[i];
        }
        if (ragged) {  // warp-uniform
            last = __shfl_sync(0xffffffffu, last, tl / per);
            for (int i = 0; i < per; ++i)
                if (lane * per + i > tl) acs[base + i] = last;
        }
    }
}

template <typename T>
static void decay_launch(dim3 grid, size_t smem, cudaStream_t st, const void *dt, const float *A_log,
                         const float *dt_bias, float dt_min, float dt_max, float *dtf, float *acs,
                         int *status, int L, int H, int chunk, int nc) {
    // at most 8 x 513 floats (chunk <= 512): under the default 48 KB, no attribute needed
    decay_prep_kernel<T><<<grid, 256, smem, st>>>((const T *)dt, A_log, dt_bias, dt_min, dt_max, dtf, acs, status,
                                                  L, H, chunk, nc);
}

cudaError_t launch_decay_prep(int dtype, const void *dt, const float *A_log, const float *dt_bias,
                              float dt_min, float dt_max, float *dtf, float *acs, int *status, int B,
                              int L, int H, int chunk, cudaStream_t st) {
    const int nc = cdiv(L, chunk);
    dim3 grid(nc, B, cdiv(H, 8));
    const size_t smem = sizeof(float) * 8 * (chunk + 1);
    if (dtype == SSD_DTYPE_BF16)
        decay_launch<__nv_bfloat16>(grid, smem, st, dt, A_log, dt_bias, dt_min, dt_max, dtf, acs, status, L, H,
                                    chunk, nc);
    else
        decay_launch<float>(grid, smem, st, dt, A_log, dt_bias, dt_min, dt_max, dtf, acs, status, L, H, chunk,
                            nc);
    return cudaGetLastError();
}

}  // namespace ssd
