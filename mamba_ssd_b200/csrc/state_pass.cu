// state_pass.cu -- step a4 of the chunked SSD: the sequential pass over chunks.
//
//   h_{-1} = h0 (or 0);   h_c = exp(acs_c[last]) * h_{c-1} + S_c
//
// in float32, in place: the chunk-state buffer S_c is overwritten with h_{c-1}, the
// state chunk c starts from, which the output correction reads next.  The state after
// the last chunk is h_final.
//
// Source: blog walk-through of "Compiler-First State Space Duality ..." (bqwf.cn) §1.1:
// chunks are computed in parallel and a light sequential scan passes the state
// between them; §3.2/§4.1: the state update stays in float32.
//
// Every (batch, head, state element) is an independent first-order recurrence, so
// the grid covers B x H x P*N/4 threads, each owning one float4 of the state and
// walking the chunks in order: fully coalesced 16-byte loads and stores, with the loads of
// eight chunks issued together so the chain costs one memory round trip per eight chunks.
// The pass is HBM/L2 bound (it touches each chunk state twice).
#include "common.cuh"
#include "launch.h"

namespace ssd {

__global__ void __launch_bounds__(256) state_pass_kernel(float *__restrict__ states,
                                                         const float *__restrict__ acs,
                                                         const float *__restrict__ h0,
                                                         float *__restrict__ h_final, int H,
                                                         int PN, int nc, int Q) {
    constexpr int kAhead = 8;  // chunk states loaded per round trip
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const size_t bh = (size_t)b * H + h;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h0) s = *reinterpret_cast<const float4 *>(h0 + bh * PN + e);
    const float *a_last = acs + bh * (size_t)nc * Q + (Q - 1);
    for (int c0 = 0; c0 < nc; c0 += kAhead) {
        float4 in[kAhead];
        float a[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            if (c0 + i < nc) {
                in[i] = *reinterpret_cast<const float4 *>(states + (((size_t)b * nc + c0 + i) * H + h) * PN + e);
                a[i] = a_last[(size_t)(c0 + i) * Q];
            }
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            if (c0 + i < nc) {
                *reinterpret_cast<float4 *>(states + (((size_t)b * nc + c0 + i) * H + h) * PN + e) = s;
                const float d = expf(a[i]);
                s.x = fmaf(d, s.x, in[i].x);
                s.y = fmaf(d, s.y, in[i].y);
                s.z = fmaf(d, s.z, in[i].z);
                s.w = fmaf(d, s.w, in[i].w);
            }
        }
    }
    if (h_final) *reinterpret_cast<float4 *>(h_final + bh * PN + e) = s;
}

cudaError_t launch_state_pass(float *states, const float *acs, const float *h0, float *h_final,
                              int B, int L, int H, int P, int N, int chunk, cudaStream_t st) {
    const int nc = cdiv(L, chunk);
    const int PN = P * N;
    dim3 grid(cdiv(PN / 4, 256), H, B);
    state_pass_kernel<<<grid, 256, 0, st>>>(states, acs, h0, h_final, H, PN, nc, chunk);
    return cudaGetLastError();
}

}  // namespace ssd
