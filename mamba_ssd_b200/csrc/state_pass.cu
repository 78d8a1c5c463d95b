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
#include "items.cuh"
#include "launch.h"
#include "tc.cuh"

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

// Variant for the tensor-core path: the block states arrive transposed, S^T [N][P] fp32 (the
// layout of the tcgen05 accumulator), and the state each block starts from is emitted in the
// same transposed layout in bf16 -- row-major [N][P], whose 128-byte-swizzled TMA tiles are the
// MN-major B operand of O = C h_prev^T -- into a separate buffer.  h0 and h_final keep the
// public [P][N] float32 layout.  Thread (n, p0..p0+3): one float4 load and one 8-byte store
// per block, consecutive threads walking p then n, so every warp access is contiguous.  Four
// blocks' loads per round trip and at most 48 registers, so five CTAs share an SM and the
// whole grid (B*H*P*N/4 threads: 640 CTAs for the 2.7B shape) is resident in one wave.
// The tensor-core workspace: block gb's decay factors of head h are the 128 floats at
// (h * nblocks + gb) * 128 (head-major), its states at (gb * H + h) * P * N (block-major).  A packed varlen batch
// (vl.n > 0) chains each sequence's own blocks, from the h0 of its index among the caller's
// sequences to that sequence's h_final; grid.z walks the sequences.
// VARLEN is a template parameter so that the equal-length instantiation carries none of the
// table lookup (it fits its 48 registers without spilling).
template <bool VARLEN>
__global__ void __launch_bounds__(256, 5) state_pass_t_kernel(const float *__restrict__ statesT,
                                                           const float *__restrict__ acs2,
                                                           const float *__restrict__ h0,
                                                           float *__restrict__ h_final,
                                                           __nv_bfloat16 *__restrict__ hT, int H,
                                                           int P, int N, int nk, int Q, int nblocks,
                                                           const Varlen vl) {
    constexpr int kAhead = 4;
    grid_dependency_wait();  // the block states come from the kernel before
    statesT = after_wait(statesT);
    acs2 = after_wait(acs2);
    h0 = after_wait(h0);
    h_final = after_wait(h_final);
    hT = after_wait(hT);
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int p0 = (t * 4) % P, n = (t * 4) / P;
    const int h = blockIdx.y;
    // (n < N for every thread of the tensor-core shape, P * N / 4 being a multiple of 256: no
    // warp is split by this exit, which the warp-wide steps below rely on)
    if (n >= N) return;
    // the sequence's first block, its block count, and where its h0 / h_final are
    int gb0 = blockIdx.z * nk, nc = nk, seq = blockIdx.z;
    if (VARLEN) {
        const int *blk0 = after_wait(vl.blk0);
        gb0 = blk0[blockIdx.z];
        nc = blk0[blockIdx.z + 1] - gb0;
        seq = after_wait(vl.seq)[blockIdx.z];
    }
    const size_t bh = (size_t)seq * H + h;
    const size_t PN = (size_t)P * N;
    float s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] = h0 ? h0[bh * PN + (size_t)(p0 + i) * N + n] : 0.f;
    // running pointers to this thread's element of block gb0 + c; consecutive blocks of one head
    // are H*P*N state elements apart (and 128 factor floats)
    const size_t step = (size_t)H * PN;
    const size_t first = ((size_t)gb0 * H + h) * PN + (size_t)n * P + p0;
    const float *src = statesT + first;
    __nv_bfloat16 *dst = hT + first;
    const float *a_last = acs2 + ((size_t)h * nblocks + gb0) * Q + (Q - 1);
    // the block states' last read: marked first to leave L2, which keeps the h_prev^T just
    // written there for the scan
    const uint64_t release = tc::l2_evict_first();
    for (int c0 = 0; c0 < nc; c0 += kAhead) {
        float4 in[kAhead];
        float a[kAhead];
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            if (c0 + j < nc) {
                in[j] = ld_global_hint(reinterpret_cast<const float4 *>(src + j * step), release);
                a[j] = a_last[j * Q];
            }
        }
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            if (c0 + j < nc) {
                __nv_bfloat162 lo2 = __floats2bfloat162_rn(s[0], s[1]);
                __nv_bfloat162 hi2 = __floats2bfloat162_rn(s[2], s[3]);
                uint2 v = make_uint2(*reinterpret_cast<uint32_t *>(&lo2), *reinterpret_cast<uint32_t *>(&hi2));
                *reinterpret_cast<uint2 *>(dst + j * step) = v;
                const float d = exp2f(a[j]);  // acs arrives as acs * log2(e) on this path
                s[0] = fmaf(d, s[0], in[j].x);
                s[1] = fmaf(d, s[1], in[j].y);
                s[2] = fmaf(d, s[2], in[j].z);
                s[3] = fmaf(d, s[3], in[j].w);
            }
        }
        // the block states just read are dead (only this pass reads them): their lines leave L2
        // without a write-back.  Every lane's loads have returned (their values are used
        // above); lanes 0, 8, 16, 24 each own one 128-byte line of the warp's 512 bytes.
        __syncwarp();
        if ((threadIdx.x & 7) == 0) {
#pragma unroll
            for (int j = 0; j < kAhead; ++j)
                if (c0 + j < nc) discard_l2_line(src + j * step);
        }
        src += kAhead * step;
        dst += kAhead * step;
        a_last += kAhead * Q;
    }
    if (h_final) {
#pragma unroll
        for (int i = 0; i < 4; ++i) h_final[bh * PN + (size_t)(p0 + i) * N + n] = s[i];
    }
    allow_dependents();
}

cudaError_t launch_state_pass_t(const float *states, const float *acs, const float *h0, float *h_final,
                                __nv_bfloat16 *hT, int B, int L, int H, int P, int N, int chunk, const Varlen &vl,
                                int nblocks, cudaStream_t st) {
    const int nk = cdiv(L, chunk);
    dim3 grid(cdiv(P * N / 4, 256), H, vl.n ? vl.n : B);
    if (vl.n)
        return launch_pdl(state_pass_t_kernel<true>, grid, dim3(256), 0, st, states, acs, h0, h_final, hT, H, P, N, nk,
                          chunk, nblocks, vl);
    return launch_pdl(state_pass_t_kernel<false>, grid, dim3(256), 0, st, states, acs, h0, h_final, hT, H, P, N, nk,
                      chunk, nblocks, vl);
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
