// chunk_simt.cu -- float32 CUDA-core versions of steps a2, a3 and a5 of the chunked SSD.
//
// These run for float32 storage, where the tolerance (relative 1e-4) leaves no room for
// bf16 or tf32 operands, and for any shape the tensor-core kernels do not cover.
//
// a3 chunk state (blog walk-through of "Compiler-First State Space Duality ..." §1.1:
//    the state each chunk passes on):
//    S_c[p][n] = sum_{s in c} dt_s * exp(acs_last - acs_s) * x_s[p] * B_s[n]
// a2 + a5 chunk scan (§1.1 decay mask L = tril(exp(segsum)), §1.2 the contraction
//    einsum('bclhn,bcshn,bhcls,bcshp->bclhp', C, B, L, X) with X = dt*x; then the
//    carried-in state and the D skip):
//    y_l[p] = sum_{s<=l} (C_l . B_s) exp(acs_l - acs_s) dt_s x_s[p]
//           + exp(acs_l) sum_n C_l[n] h_prev[p][n] + D x_l[p]
//
// The head dimension P is 64.  Each CTA computes a 64-wide tile with 256 threads in a
// 16 x 16 grid of 4 x 4 (or 4 x N/16) register micro-tiles; operands are staged in
// shared memory, transposed so that every inner-loop read is a 16-byte vector.
// exp(acs_l - acs_s) is taken only where s <= l (masked before the exp, never as a
// ratio of two exponentials), so nothing overflows.
#include "common.cuh"
#include "launch.h"

namespace ssd {

constexpr int kP = 64;  // head dimension handled by these kernels

// ------------------------------------------------------------------------------------
// a3: chunk state.  grid (nc, H, B), 256 threads.  Thread (ty, tx) owns p = 4ty..4ty+3
// and n = tx*NPT .. tx*NPT+NPT-1.
// ------------------------------------------------------------------------------------
template <typename T, int N>
__global__ void __launch_bounds__(256) chunk_state_simt_kernel(
    const T *__restrict__ x, const T *__restrict__ Bm, const float *__restrict__ dtf,
    const float *__restrict__ acs, float *__restrict__ states, int L, int H, int G, int Q,
    int nc, int64_t x_row, int64_t bc_row) {
    constexpr int NPT = N / 16;
    constexpr int SB = 32;  // tokens per stage
    __shared__ __align__(16) float Xs[SB][kP];
    __shared__ __align__(16) float Bs[SB][N];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const size_t Lp = (size_t)nc * Q;
    const float *dt_row = dtf + ((size_t)b * H + h) * Lp + (size_t)c * Q;
    const float *acs_row = acs + ((size_t)b * H + h) * Lp + (size_t)c * Q;
    const float a_last = acs_row[Q - 1];

    float acc[4][NPT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NPT; ++j) acc[i][j] = 0.f;

    for (int s0 = 0; s0 < Q; s0 += SB) {
        for (int idx = tid; idx < SB * kP; idx += 256) {
            const int s = idx / kP, p = idx % kP;
            const int tok = c * Q + s0 + s;
            float v = 0.f;
            if (tok < L) {
                const float w = dt_row[s0 + s] * expf(a_last - acs_row[s0 + s]);
                v = w * to_f(x[((size_t)b * L + tok) * x_row + (size_t)h * kP + p]);
            }
            Xs[s][p] = v;
        }
        for (int idx = tid; idx < SB * N; idx += 256) {
            const int s = idx / N, n = idx % N;
            const int tok = c * Q + s0 + s;
            Bs[s][n] = tok < L ? to_f(Bm[((size_t)b * L + tok) * bc_row + (size_t)g * N + n]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < SB; ++s) {
            const float4 a4 = *reinterpret_cast<const float4 *>(&Xs[s][ty * 4]);
            float bv[NPT];
#pragma unroll
            for (int j = 0; j < NPT; ++j) bv[j] = Bs[s][tx * NPT + j];
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < NPT; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float *out = states + (((size_t)b * nc + c) * H + h) * (size_t)kP * N;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NPT; ++j) out[(size_t)(ty * 4 + i) * N + tx * NPT + j] = acc[i][j];
}

// ------------------------------------------------------------------------------------
// a2 + a5: chunk scan.  grid (nc * Q/64, H, B), 256 threads; the CTA owns 64 rows l of
// one chunk and all 64 columns p.  Thread (ty, tx) owns l = 4ty.., p = 4tx.. .
// Shared memory (floats): Cs[N][68], Bs[N][68] (reused for h_prev^T), Ps[64][68],
// Xs[64][68], plus the cumsums of the row block and of the column block.
// ------------------------------------------------------------------------------------
constexpr int kLd = 68;  // padded row length (keeps 16-byte alignment, spreads banks)

template <int N>
constexpr size_t chunk_scan_simt_smem() {
    return sizeof(float) * (2 * (size_t)N * kLd + 2 * 64 * kLd + 2 * 64);
}

template <typename T, int N>
__global__ void __launch_bounds__(256) chunk_scan_simt_kernel(
    const T *__restrict__ x, const T *__restrict__ Bm, const T *__restrict__ Cm,
    const float *__restrict__ dtf, const float *__restrict__ acs, const float *__restrict__ hprev,
    const float *__restrict__ D, T *__restrict__ y, int L, int H, int G, int Q, int nc, int64_t x_row,
    int64_t bc_row) {
    extern __shared__ __align__(16) float smem[];
    float *Cs = smem;                  // [N][kLd]   C rows of the row block, transposed
    float *Bs = Cs + N * kLd;          // [N][kLd]   B rows of a column block, transposed
    float *Ps = Bs + N * kLd;          // [64][kLd]  masked decay-weighted C.B, [s][l]
    float *Xs = Ps + 64 * kLd;         // [64][kLd]  dt_s * x_s[p], [s][p]
    float *acs_l = Xs + 64 * kLd;      // [64]
    float *acs_s = acs_l + 64;         // [64]

    const int blocks_per_chunk = Q / 64;
    const int c = blockIdx.x / blocks_per_chunk, lb = blockIdx.x % blocks_per_chunk;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const size_t Lp = (size_t)nc * Q;
    const float *dt_row = dtf + ((size_t)b * H + h) * Lp + (size_t)c * Q;
    const float *acs_row = acs + ((size_t)b * H + h) * Lp + (size_t)c * Q;
    const int l0 = lb * 64;  // first row of this block inside the chunk

    for (int idx = tid; idx < 64 * N; idx += 256) {
        const int l = idx / N, n = idx % N;
        const int tok = c * Q + l0 + l;
        Cs[n * kLd + l] = tok < L ? to_f(Cm[((size_t)b * L + tok) * bc_row + (size_t)g * N + n]) : 0.f;
    }
    if (tid < 64) acs_l[tid] = acs_row[l0 + tid];

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // ---- intra-chunk part: column blocks up to and including the diagonal block ----
    for (int sb = 0; sb <= lb; ++sb) {
        const int s0 = sb * 64;
        __syncthreads();  // previous Bs / Ps / Xs reads are done
        for (int idx = tid; idx < 64 * N; idx += 256) {
            const int s = idx / N, n = idx % N;
            const int tok = c * Q + s0 + s;
            Bs[n * kLd + s] = tok < L ? to_f(Bm[((size_t)b * L + tok) * bc_row + (size_t)g * N + n]) : 0.f;
        }
        for (int idx = tid; idx < 64 * kP; idx += 256) {
            const int s = idx / kP, p = idx % kP;
            const int tok = c * Q + s0 + s;
            Xs[s * kLd + p] =
                tok < L ? dt_row[s0 + s] * to_f(x[((size_t)b * L + tok) * x_row + (size_t)h * kP + p]) : 0.f;
        }
        if (tid < 64) acs_s[tid] = acs_row[s0 + tid];
        __syncthreads();
        // CB micro-tile: rows l = 4ty+i, columns s = 4tx+j
        float cb[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) cb[i][j] = 0.f;
#pragma unroll 4
        for (int n = 0; n < N; ++n) {
            const float4 c4 = *reinterpret_cast<const float4 *>(&Cs[n * kLd + ty * 4]);
            const float4 b4 = *reinterpret_cast<const float4 *>(&Bs[n * kLd + tx * 4]);
            const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
            const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) cb[i][j] = fmaf(cv[i], bv[j], cb[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int l = ty * 4 + i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s = tx * 4 + j;
                const bool keep = (sb < lb) || (s <= l);
                Ps[s * kLd + l] = keep ? cb[i][j] * expf(acs_l[l] - acs_s[s]) : 0.f;
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < 64; ++s) {
            const float4 p4 = *reinterpret_cast<const float4 *>(&Ps[s * kLd + ty * 4]);
            const float4 x4 = *reinterpret_cast<const float4 *>(&Xs[s * kLd + tx * 4]);
            const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
            const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(pv[i], xv[j], acc[i][j]);
        }
    }

    // ---- carried-in state: exp(acs_l) * sum_n C_l[n] h_prev[p][n] ----
    __syncthreads();
    const float *hp = hprev + (((size_t)b * nc + c) * H + h) * (size_t)kP * N;
    for (int idx = tid; idx < kP * N; idx += 256) {
        const int p = idx / N, n = idx % N;
        Bs[n * kLd + p] = hp[idx];
    }
    __syncthreads();
    float off[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) off[i][j] = 0.f;
#pragma unroll 4
    for (int n = 0; n < N; ++n) {
        const float4 c4 = *reinterpret_cast<const float4 *>(&Cs[n * kLd + ty * 4]);
        const float4 h4 = *reinterpret_cast<const float4 *>(&Bs[n * kLd + tx * 4]);
        const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
        const float hv[4] = {h4.x, h4.y, h4.z, h4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) off[i][j] = fmaf(cv[i], hv[j], off[i][j]);
    }

    // ---- epilogue: y = diag + exp(acs_l) * off + D x ----
    const float d = D ? D[h] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int l = ty * 4 + i;
        const int tok = c * Q + l0 + l;
        if (tok >= L) continue;
        const float e = expf(acs_l[l]);
        const size_t rowoff = (((size_t)b * L + tok) * H + h) * kP;  // y is dense
        const size_t xoff = ((size_t)b * L + tok) * x_row + (size_t)h * kP;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = tx * 4 + j;
            const float xv = to_f(x[xoff + p]);
            y[rowoff + p] = from_f<T>(acc[i][j] + e * off[i][j] + d * xv);
        }
    }
}

template <typename T, int N>
static cudaError_t chunk_state_n(const void *x, const void *Bm, const float *dtf, const float *acs,
                                 float *states, int B, int L, int H, int G, int chunk, int64_t x_row,
                                 int64_t bc_row, cudaStream_t st) {
    const int nc = cdiv(L, chunk);
    dim3 grid(nc, H, B);
    chunk_state_simt_kernel<T, N><<<grid, 256, 0, st>>>((const T *)x, (const T *)Bm, dtf, acs,
                                                        states, L, H, G, chunk, nc, x_row, bc_row);
    return cudaGetLastError();
}

template <typename T, int N>
static cudaError_t chunk_scan_n(const void *x, const void *Bm, const void *Cm, const float *dtf,
                                const float *acs, const float *hprev, const float *D, void *y,
                                int B, int L, int H, int G, int chunk, int64_t x_row, int64_t bc_row,
                                cudaStream_t st) {
    const int nc = cdiv(L, chunk);
    dim3 grid(nc * (chunk / 64), H, B);
    constexpr size_t smem = chunk_scan_simt_smem<N>();
    const cudaError_t e = raise_smem_limit<chunk_scan_simt_kernel<T, N>>((int)smem);
    if (e != cudaSuccess) return e;
    chunk_scan_simt_kernel<T, N><<<grid, 256, smem, st>>>((const T *)x, (const T *)Bm,
                                                          (const T *)Cm, dtf, acs, hprev, D,
                                                          (T *)y, L, H, G, chunk, nc, x_row, bc_row);
    return cudaGetLastError();
}

#define SSD_DISPATCH_N(N, FN, T, ...)                            \
    switch (N) {                                                 \
        case 16: return FN<T, 16>(__VA_ARGS__);                  \
        case 32: return FN<T, 32>(__VA_ARGS__);                  \
        case 64: return FN<T, 64>(__VA_ARGS__);                  \
        case 128: return FN<T, 128>(__VA_ARGS__);                \
        default: return cudaErrorInvalidValue;                   \
    }

cudaError_t launch_chunk_state(int dtype, const void *x, const void *Bm, const float *dtf,
                               const float *acs, float *states, int B, int L, int H, int G, int N,
                               int chunk, int64_t x_row, int64_t bc_row, cudaStream_t st) {
    if (dtype == SSD_DTYPE_BF16) {
        SSD_DISPATCH_N(N, chunk_state_n, __nv_bfloat16, x, Bm, dtf, acs, states, B, L, H, G, chunk, x_row, bc_row,
                       st)
    }
    SSD_DISPATCH_N(N, chunk_state_n, float, x, Bm, dtf, acs, states, B, L, H, G, chunk, x_row, bc_row, st)
}

cudaError_t launch_chunk_scan(int dtype, const void *x, const void *Bm, const void *Cm,
                              const float *dtf, const float *acs, const float *hprev,
                              const float *D, void *y, int B, int L, int H, int G, int N,
                              int chunk, int64_t x_row, int64_t bc_row, cudaStream_t st) {
    if (dtype == SSD_DTYPE_BF16) {
        SSD_DISPATCH_N(N, chunk_scan_n, __nv_bfloat16, x, Bm, Cm, dtf, acs, hprev, D, y, B, L, H,
                       G, chunk, x_row, bc_row, st)
    }
    SSD_DISPATCH_N(N, chunk_scan_n, float, x, Bm, Cm, dtf, acs, hprev, D, y, B, L, H, G, chunk, x_row, bc_row,
                   st)
}

}  // namespace ssd
