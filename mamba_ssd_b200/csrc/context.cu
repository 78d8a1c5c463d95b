// context.cu -- the two small steps of a context-parallel prefill, where the sequence is split
// into W consecutive segments (one per GPU) and each segment's scan needs the state the
// segments before it leave.
//
// The recurrence h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T is linear in h, so a segment maps
// its incoming state h_in to exp(sum_{t in seg} dt_t A) h_in + S_seg, where S_seg is the state
// the segment leaves when it starts from zero (ssd_chunk_scan_fwd with y = NULL computes it).
// Source: the blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §1.1: the state passed between chunks, with
// a light sequential scan between them -- here the chunks are whole segments on different
// GPUs, and the scan between them runs after one exchange of (S_seg, decay).
//
//   segment_decay_kernel:  log2 of each (batch, head) segment's total decay,
//                          A_h * sum_t clip(softplus(dt_t + dt_bias_h)) * log2(e)
//   state_combine_kernel:  h = h0 (or 0); for j < r: h = exp2(ld_j) h + S_j; out = h
//                          (the carry-in of segment r, or with r = W the state after the
//                          whole sequence)
#include "common.cuh"
#include "launch.h"

namespace ssd {

// One CTA of 256 threads per (batch, 32 heads): lane = head, warp = a slice of the tokens; the
// warps' partial sums meet in shared memory.  dt rows are read 32 heads wide, coalesced.
template <typename T>
__global__ void __launch_bounds__(256) segment_decay_kernel(const T *__restrict__ dt, const float *__restrict__ A_log,
                                                            const float *__restrict__ dt_bias, float dt_min,
                                                            float dt_max, float *__restrict__ out, int L, int H) {
    __shared__ float part[8][33];
    const int b = blockIdx.x, h = blockIdx.y * 32 + (threadIdx.x & 31), warp = threadIdx.x >> 5;
    float sum = 0.f;
    if (h < H) {
        const float bias = dt_bias ? dt_bias[h] : 0.f;
        for (int t = warp; t < L; t += 8)
            sum += discretise_dt(to_f(dt[((size_t)b * L + t) * H + h]), bias, dt_min, dt_max);
    }
    part[warp][threadIdx.x & 31] = sum;
    __syncthreads();
    if (warp == 0 && h < H) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += part[w][threadIdx.x];
        out[(size_t)b * H + h] = -expf(A_log[h]) * s * kLog2e;
    }
}

// One thread per float4 of the [B, H, P, N] state.
__global__ void __launch_bounds__(256) state_combine_kernel(const float *__restrict__ states,
                                                            const float *__restrict__ log2_decays,
                                                            const float *__restrict__ h0, float *__restrict__ out,
                                                            int r, size_t n4, int PN4, int BH) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const int bh = (int)(i / PN4);
    float4 h = h0 ? reinterpret_cast<const float4 *>(h0)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < r; ++j) {
        const float a = exp2f(log2_decays[(size_t)j * BH + bh]);
        const float4 s = reinterpret_cast<const float4 *>(states)[(size_t)j * n4 + i];
        h.x = fmaf(a, h.x, s.x);
        h.y = fmaf(a, h.y, s.y);
        h.z = fmaf(a, h.z, s.z);
        h.w = fmaf(a, h.w, s.w);
    }
    reinterpret_cast<float4 *>(out)[i] = h;
}

cudaError_t launch_segment_decay(int dtype, const void *dt, const float *A_log, const float *dt_bias, float dt_min,
                                 float dt_max, float *out, int B, int L, int H, cudaStream_t st) {
    dim3 grid(B, cdiv(H, 32));
    if (dtype == SSD_DTYPE_BF16)
        segment_decay_kernel<__nv_bfloat16>
            <<<grid, 256, 0, st>>>((const __nv_bfloat16 *)dt, A_log, dt_bias, dt_min, dt_max, out, L, H);
    else
        segment_decay_kernel<float><<<grid, 256, 0, st>>>((const float *)dt, A_log, dt_bias, dt_min, dt_max, out, L, H);
    return cudaGetLastError();
}

cudaError_t launch_state_combine(const float *states, const float *log2_decays, const float *h0, float *out, int r,
                                 int B, int H, int P, int N, cudaStream_t st) {
    const size_t n4 = (size_t)B * H * P * N / 4;
    const int threads = 256;
    const size_t blocks = (n4 + threads - 1) / threads;
    state_combine_kernel<<<(unsigned)blocks, threads, 0, st>>>(states, log2_decays, h0, out, r, n4, P * N / 4, B * H);
    return cudaGetLastError();
}

}  // namespace ssd
