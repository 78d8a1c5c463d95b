// run_pass.cu -- second kernel of the fused tensor-core prefill: the inter-chunk state pass
// (step a4) over runs instead of blocks.
//
//   h = h0 (or 0);  for each run r of the chain, in order:  carry_in(r) = h;
//                                                            h = exp2(decay_r) h + S_r
//   h_final = h
//
// where S_r and decay_r are the run's own state and total decay from run_state_tc (a run
// chains its blocks' states exactly as the blocks chain into the run: the recurrence is
// linear).  Each run's slot is overwritten in place by the state the run starts from, which
// the fused scan reads.  Source: blog walk-through of "Compiler-First State Space Duality and
// Portable O(1) Autoregressive Caching for Inference" (bqwf.cn) §1.1 (the light sequential
// scan between chunks) and §3.2 / §4.1 (the state update in float32).
//
// One CTA of 256 threads per (chain, head): a thread owns 8 float4 of the head's [N][P]
// state; the runs of a chain are found from the CTA ranges of runs.cuh (at most a few per
// chain at the workloads' sizes), each run's state loaded while the previous run's carry-in
// is written.  h0 and h_final keep the public [P][N] layout, transposed through shared memory.
#include "common.cuh"
#include "launch.h"
#include "runs.cuh"

namespace ssd {

__global__ void __launch_bounds__(256) run_pass_kernel(float *__restrict__ slots, const float *__restrict__ decays,
                                                       const float *__restrict__ h0, float *__restrict__ h_final,
                                                       int H, RunLayout lay) {
    constexpr int P = 64, N = 128, kPer = P * N / 4 / 256;  // float4 per thread: 8
    constexpr int kLd = P + 1;                               // padded [N][P + 1] transpose tile
    __shared__ float tile[N * kLd];
    grid_dependency_wait();  // the run states come from the kernel before
    slots = after_wait(slots);
    decays = after_wait(decays);
    h0 = after_wait(h0);
    h_final = after_wait(h_final);
    const int ch = blockIdx.x, hh = blockIdx.y;
    const int NQ = H / kPairHeads;
    const int b = ch / NQ, h = (ch - b * NQ) * kPairHeads + hh;
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x;
    // the public [P][N] layout of h0 and h_final goes through the tile, so that both global
    // sides are read and written along n, contiguously
    float4 s[kPer];
    if (h0) {
        for (int idx = tid; idx < P * N; idx += 256) tile[(idx % N) * kLd + idx / N] = h0[bh * P * N + idx];
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = (tid + 256 * i) * 4;  // element (n, p) = (e / P, e % P) of [N][P]
        const float *t = tile + (e / P) * kLd + e % P;
        s[i] = h0 ? make_float4(t[0], t[1], t[2], t[3]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int u_first = ch * lay.nk, u_last = u_first + lay.nk - 1;
    const int c_lo = lay.cta_of(u_first), c_hi = lay.cta_of(u_last);
    auto slot_ptr = [&](int c) {
        const int slot = c == c_lo ? ch : lay.nch + c;
        return reinterpret_cast<float4 *>(slots + ((size_t)slot * kPairHeads + hh) * P * N);
    };
    auto slot_decay = [&](int c) { return decays[(c == c_lo ? ch : lay.nch + c) * kPairHeads + hh]; };
    float4 nxt[kPer];
    float a_nxt = slot_decay(c_lo);
    {
        const float4 *st = slot_ptr(c_lo);
#pragma unroll
        for (int i = 0; i < kPer; ++i) nxt[i] = st[tid + 256 * i];
    }
    for (int c = c_lo; c <= c_hi; ++c) {
        float4 in[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) in[i] = nxt[i];
        const float a = exp2f(a_nxt);
        if (c < c_hi) {  // the next run's state, in flight while this run's carry-in is written
            const float4 *st = slot_ptr(c + 1);
            a_nxt = slot_decay(c + 1);
#pragma unroll
            for (int i = 0; i < kPer; ++i) nxt[i] = st[tid + 256 * i];
        }
        float4 *st = slot_ptr(c);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            st[tid + 256 * i] = s[i];
            s[i].x = fmaf(a, s[i].x, in[i].x);
            s[i].y = fmaf(a, s[i].y, in[i].y);
            s[i].z = fmaf(a, s[i].z, in[i].z);
            s[i].w = fmaf(a, s[i].w, in[i].w);
        }
    }
    if (h_final) {
        __syncthreads();  // every thread is done reading the tile (h0)
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = (tid + 256 * i) * 4;
            float *t = tile + (e / P) * kLd + e % P;
            t[0] = s[i].x;
            t[1] = s[i].y;
            t[2] = s[i].z;
            t[3] = s[i].w;
        }
        __syncthreads();
        for (int idx = tid; idx < P * N; idx += 256) h_final[bh * P * N + idx] = tile[(idx % N) * kLd + idx / N];
    }
    allow_dependents();
}

cudaError_t launch_run_pass(float *slots, const float *decays, const float *h0, float *h_final, int B, int H,
                            const RunLayout &lay, cudaStream_t st) {
    dim3 grid(B * (H / kPairHeads), kPairHeads);
    return launch_pdl(run_pass_kernel, grid, dim3(256), 0, st, slots, decays, h0, h_final, H, lay);
}

}  // namespace ssd
