// gated_rmsnorm.cu -- the block step after the scan: y * SiLU(z), RMS-normalised per token
// and norm group, scaled per channel.
//
//   g   = y * SiLU(z)
//   out = g / sqrt(mean over the group's channels of g^2 + eps) * w
//
// Source: the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §4.1 (a norm takes its
// variance in float32 even for bf16 inputs) and §3.2 (norms sit next to the SSD and are fused
// into their neighbours); the gate and the per-group RMS are the Mamba-2 block's norm, which
// the pages name but do not spell out.
//
// HBM-bound: 3 * GS * sizeof(T) bytes per (token, group) row, plus w, which stays in L2.  Three
// forms, none with a spin-wait of any kind:
//
// Warp streaming form (rows of at most 128 16-byte vectors: up to 1024 bf16 or 512 float32
// channels per group).  As the streaming form below, with a warp in place of a CTA: each warp
// walks its own rows, through its own slice of the ring, holding up to 4 vectors of y and of z
// per lane, and sums the squares with shuffles, so nothing waits on another warp.
//
// Streaming form (a group's y row at most 20 KB: up to 10240 bf16 or 5120 float32 channels).
// Persistent CTAs, as many as fit on the GPU at once, each walking rows gridDim.x apart.  A
// thread owns 16 elements of a row (GS / 16 threads, rounded up to a warp).  While it works
// on row k it has already asked for its 16-byte vectors of y and z of row k + 1: cp.async
// copies them into the other half of a two-stage shared-memory ring.  Each thread reads back
// only the vectors it copied itself, so waiting on its own copies (cp.async.wait_group) is
// all the ordering the data needs; the one CTA barrier per row is the sum of squares.  A CTA
// therefore always has a row of loads in flight, also while it reduces and stores.
//
// Staged form (larger groups, up to 32768 channels).  One CTA per (token, norm group).  The
// group's GS channels stream in once as 16-byte vectors of y and z; each thread keeps its gated
// values in shared memory (fp32) and adds up their squares in fp32; the CTA reduces the sum,
// and a second pass over shared memory scales by the reciprocal RMS and by w and streams the
// result out.
#include "common.cuh"
#include "launch.h"
#include "stream.cuh"
#include "tc.cuh"

namespace ssd {

constexpr int kNormThreads = 256;
constexpr int kNormMaxGroup = 32768;  // channels per norm group: 128 KB of staged fp32
constexpr int kNormBatch = 3;         // 16-byte vectors of y and of z in flight per thread

template <typename T>
struct Vec16;  // 16 bytes of T
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
};
template <>
struct Vec16<float> {
    static constexpr int n = 4;
};

template <typename T>
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(const T *__restrict__ y,
                                                                     const T *__restrict__ z,
                                                                     const float *__restrict__ w,
                                                                     T *__restrict__ out, int C, int GS,
                                                                     float eps) {
    extern __shared__ __align__(16) float g_s[];  // [GS] gated values of this row
    __shared__ float red[kNormThreads / 32];
    constexpr int VEC = Vec16<T>::n;

    grid_dependency_wait();  // y comes from the kernel before
    y = after_wait(y);
    z = after_wait(z);
    w = after_wait(w);
    out = after_wait(out);

    const size_t base = (size_t)blockIdx.x * C + (size_t)blockIdx.y * GS;
    const int nvec = GS / VEC;
    const uint4 *y4 = reinterpret_cast<const uint4 *>(y + base);
    const uint4 *z4 = reinterpret_cast<const uint4 *>(z + base);

    // ---- pass 1: gate, stage, sum of squares (fp32).  A thread's vectors of a batch are all
    // requested before any is used, so a row costs one memory round trip, not one per vector.
    float ss = 0.f;
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kNormBatch * kNormThreads) {
        uint4 yr[kNormBatch], zr[kNormBatch];
#pragma unroll
        for (int i = 0; i < kNormBatch; ++i) {
            const int v = v0 + i * kNormThreads;
            if (v < nvec) {
                yr[i] = __ldcs(y4 + v);  // read once: evict first
                zr[i] = __ldcs(z4 + v);
            }
        }
#pragma unroll
        for (int i = 0; i < kNormBatch; ++i) {
            const int v = v0 + i * kNormThreads;
            if (v < nvec) {
                const T *ye = reinterpret_cast<const T *>(&yr[i]);
                const T *ze = reinterpret_cast<const T *>(&zr[i]);
                float g[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    g[e] = to_f(ye[e]) * silu_fast(to_f(ze[e]));
                    ss = fmaf(g[e], g[e], ss);
                }
                float4 *dst = reinterpret_cast<float4 *>(g_s + v * VEC);
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q)
                    dst[q] = make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
            }
        }
    }
    // ---- CTA sum ----
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) tot += red[i];
    const float rinv = 1.f / sqrtf(tot / (float)GS + eps);

    // ---- pass 2: scale and store (each thread re-reads only what it staged) ----
    const float4 *w4 = reinterpret_cast<const float4 *>(w + (size_t)blockIdx.y * GS);
    uint4 *o4 = reinterpret_cast<uint4 *>(out + base);
    for (int v = threadIdx.x; v < nvec; v += kNormThreads) {
        const float4 *src = reinterpret_cast<const float4 *>(g_s + v * VEC);
        uint4 packed;
        T *oe = reinterpret_cast<T *>(&packed);
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
            const float4 g = src[q];
            const float4 wv = __ldg(w4 + v * (VEC / 4) + q);
            oe[4 * q + 0] = from_f<T>(g.x * rinv * wv.x);
            oe[4 * q + 1] = from_f<T>(g.y * rinv * wv.y);
            oe[4 * q + 2] = from_f<T>(g.z * rinv * wv.z);
            oe[4 * q + 3] = from_f<T>(g.w * rinv * wv.w);
        }
        __stcs(o4 + v, packed);
    }
    allow_dependents();
}

constexpr int kNormStreamElems = 16;          // elements of a row per thread
constexpr int kNormStreamRowBytes = 20480;    // largest y (or z) row of one group
constexpr int kNormStreamMaxThreads = kNormStreamRowBytes / 2 / kNormStreamElems;  // bf16: 640

// rows: T_rows * n_groups (token-major, group fastest).  blockDim.x * VPT * VEC >= GS.
template <typename T>
__global__ void __launch_bounds__(kNormStreamMaxThreads) gated_rmsnorm_stream_kernel(
    const T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w, T *__restrict__ out, int C,
    int GS, int n_groups, int rows, float eps) {
    constexpr int VEC = Vec16<T>::n;
    constexpr int VPT = kNormStreamElems / VEC;  // 16-byte vectors of y (and of z) per thread
    extern __shared__ __align__(16) uint4 ring_s[];  // [2 stages][y, z][GS / VEC vectors]
    __shared__ __align__(16) float red[2][kNormStreamMaxThreads / 32];  // zero past the last warp

    const int nthr = blockDim.x;
    const int nwarp4 = ((nthr >> 5) + 3) & ~3;  // warps rounded up to a float4 of red
    if (threadIdx.x < 2 * nwarp4) red[threadIdx.x / nwarp4][threadIdx.x % nwarp4] = 0.f;

    grid_dependency_wait();  // y comes from the kernel before
    y = after_wait(y);
    z = after_wait(z);
    w = after_wait(w);
    out = after_wait(out);

    const int nvec = GS / VEC;
    const uint64_t first = tc::l2_evict_first();  // y and z are read once

    // Rows r = t * n_groups + gi advance by gridDim.x = dt * n_groups + dg, so (t, gi) step by
    // additions instead of divisions.
    const int dt = gridDim.x / n_groups, dg = gridDim.x - dt * n_groups;
    auto step = [&](int &t, int &gi) {
        t += dt;
        gi += dg;
        if (gi >= n_groups) {
            gi -= n_groups;
            ++t;
        }
    };

    // this thread's vectors of row (t, gi) into stage s; always one commit group per call
    auto request = [&](int r, int t, int gi, int s) {
        if (r < rows) {
            const size_t base = (size_t)t * C + (size_t)gi * GS;
            const uint4 *y4 = reinterpret_cast<const uint4 *>(y + base);
            const uint4 *z4 = reinterpret_cast<const uint4 *>(z + base);
            uint4 *sy = ring_s + (size_t)s * 2 * nvec;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = threadIdx.x + i * nthr;
                if (v < nvec) {
                    cp_async16(sy + v, y4 + v, first);
                    cp_async16(sy + nvec + v, z4 + v, first);
                }
            }
        }
        cp_async_commit();
    };

    int r = blockIdx.x;
    int t = r / n_groups, gi = r - t * n_groups;  // row r's token and group
    int tn = t, gn = gi;                          // those of row r + gridDim.x
    step(tn, gn);
    __syncthreads();  // red's zero padding
    request(r, t, gi, 0);
    for (int k = 0; r < rows; ++k, r += gridDim.x) {
        request(r + gridDim.x, tn, gn, (k + 1) & 1);
        cp_async_wait<1>();  // every group but the newest: row r's copies have landed

        // ---- gate and sum of squares (fp32), from the vectors this thread copied ----
        const uint4 *sy = ring_s + (size_t)(k & 1) * 2 * nvec;
        float g[VPT][VEC];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = threadIdx.x + i * nthr;
            if (v < nvec) {
                const uint4 yr = sy[v], zr = sy[nvec + v];
                const T *ye = reinterpret_cast<const T *>(&yr);
                const T *ze = reinterpret_cast<const T *>(&zr);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    g[i][e] = to_f(ye[e]) * silu_ftz(to_f(ze[e]));
                    ss = fmaf(g[i][e], g[i][e], ss);
                }
            }
        }
        // ---- CTA sum: red alternates between two halves, so one barrier per row suffices ----
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((threadIdx.x & 31) == 0) red[k & 1][threadIdx.x >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
        const float4 *red4 = reinterpret_cast<const float4 *>(red[k & 1]);
        for (int i = 0; i < (nwarp4 >> 2); ++i) {
            const float4 q = red4[i];
            tot += (q.x + q.y) + (q.z + q.w);
        }
        const float rinv = rsqrtf(tot / (float)GS + eps);

        // ---- scale and store ----
        const float4 *w4 = reinterpret_cast<const float4 *>(w + (size_t)gi * GS);
        uint4 *o4 = reinterpret_cast<uint4 *>(out + (size_t)t * C + (size_t)gi * GS);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = threadIdx.x + i * nthr;
            if (v < nvec) {
                uint4 packed;
                T *oe = reinterpret_cast<T *>(&packed);
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q) {
                    const float4 wv = __ldg(w4 + v * (VEC / 4) + q);
                    oe[4 * q + 0] = from_f<T>(g[i][4 * q + 0] * rinv * wv.x);
                    oe[4 * q + 1] = from_f<T>(g[i][4 * q + 1] * rinv * wv.y);
                    oe[4 * q + 2] = from_f<T>(g[i][4 * q + 2] * rinv * wv.z);
                    oe[4 * q + 3] = from_f<T>(g[i][4 * q + 3] * rinv * wv.w);
                }
                __stcs(o4 + v, packed);
            }
        }
        t = tn;
        gi = gn;
        step(tn, gn);
    }
    allow_dependents();
}

constexpr int kNormWarpThreads = 256;
constexpr int kNormWarpMaxVec = 4;  // 16-byte vectors of y (and of z) per lane

// rows: T_rows * n_groups (token-major, group fastest).  32 * VPT * VEC >= GS.
template <typename T, int VPT>
__global__ void __launch_bounds__(kNormWarpThreads) gated_rmsnorm_warp_kernel(
    const T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w, T *__restrict__ out, int C,
    int GS, int n_groups, int rows, float eps) {
    constexpr int VEC = Vec16<T>::n;
    constexpr int WARPS = kNormWarpThreads / 32;
    extern __shared__ __align__(16) uint4 ring_s[];  // [WARPS][2 stages][y, z][GS / VEC vectors]

    grid_dependency_wait();  // y comes from the kernel before
    y = after_wait(y);
    z = after_wait(z);
    w = after_wait(w);
    out = after_wait(out);

    const int nvec = GS / VEC;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint4 *ring = ring_s + (size_t)wib * 4 * nvec;  // this warp's two stages
    const uint64_t first = tc::l2_evict_first();    // y and z are read once

    // rows r = t * n_groups + gi advance by the number of warps in the grid
    const int nw = gridDim.x * WARPS;
    const int dt = nw / n_groups, dg = nw - dt * n_groups;
    auto step = [&](int &t, int &gi) {
        t += dt;
        gi += dg;
        if (gi >= n_groups) {
            gi -= n_groups;
            ++t;
        }
    };
    // this lane's vectors of row (t, gi) into stage s; always one commit group per call
    auto request = [&](int r, int t, int gi, int s) {
        if (r < rows) {
            const size_t base = (size_t)t * C + (size_t)gi * GS;
            const uint4 *y4 = reinterpret_cast<const uint4 *>(y + base);
            const uint4 *z4 = reinterpret_cast<const uint4 *>(z + base);
            uint4 *sy = ring + (size_t)s * 2 * nvec;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + i * 32;
                if (v < nvec) {
                    cp_async16(sy + v, y4 + v, first);
                    cp_async16(sy + nvec + v, z4 + v, first);
                }
            }
        }
        cp_async_commit();
    };

    int r = blockIdx.x * WARPS + wib;
    int t = r / n_groups, gi = r - t * n_groups;
    int tn = t, gn = gi;
    step(tn, gn);
    request(r, t, gi, 0);
    for (int k = 0; r < rows; ++k, r += nw) {
        request(r + nw, tn, gn, (k + 1) & 1);
        cp_async_wait<1>();  // every group but the newest: row r's copies have landed

        const uint4 *sy = ring + (size_t)(k & 1) * 2 * nvec;
        float g[VPT][VEC];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + i * 32;
            if (v < nvec) {
                const uint4 yr = sy[v], zr = sy[nvec + v];
                const T *ye = reinterpret_cast<const T *>(&yr);
                const T *ze = reinterpret_cast<const T *>(&zr);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    g[i][e] = to_f(ye[e]) * silu_ftz(to_f(ze[e]));
                    ss = fmaf(g[i][e], g[i][e], ss);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // every lane: the row's sum
        const float rinv = rsqrtf(ss / (float)GS + eps);

        const float4 *w4 = reinterpret_cast<const float4 *>(w + (size_t)gi * GS);
        uint4 *o4 = reinterpret_cast<uint4 *>(out + (size_t)t * C + (size_t)gi * GS);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + i * 32;
            if (v < nvec) {
                uint4 packed;
                T *oe = reinterpret_cast<T *>(&packed);
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q) {
                    const float4 wv = __ldg(w4 + v * (VEC / 4) + q);
                    oe[4 * q + 0] = from_f<T>(g[i][4 * q + 0] * rinv * wv.x);
                    oe[4 * q + 1] = from_f<T>(g[i][4 * q + 1] * rinv * wv.y);
                    oe[4 * q + 2] = from_f<T>(g[i][4 * q + 2] * rinv * wv.z);
                    oe[4 * q + 3] = from_f<T>(g[i][4 * q + 3] * rinv * wv.w);
                }
                __stcs(o4 + v, packed);
            }
        }
        t = tn;
        gi = gn;
        step(tn, gn);
    }
    allow_dependents();
}

template <typename T, int VPT>
static cudaError_t norm_warp_launch(const void *y, const void *z, const float *w, void *out, int T_rows, int C,
                                    int n_groups, float eps, cudaStream_t st) {
    constexpr auto kernel = gated_rmsnorm_warp_kernel<T, VPT>;
    constexpr int kWarps = kNormWarpThreads / 32;
    const int GS = C / n_groups;
    const int smem = kWarps * 2 * 2 * GS * (int)sizeof(T);  // at most 64 KB
    const int rows = T_rows * n_groups;                     // below 2^30 (the dispatcher's rule)
    cudaError_t e = raise_smem_limit<kernel>(kWarps * 2 * 2 * kNormWarpMaxVec * 32 * 16);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kNormWarpThreads, smem)) != cudaSuccess)
        return e;
    if (per_sm < 1) per_sm = 1;
    const long long resident = (long long)sms * per_sm;
    const long long need = (rows + kWarps - 1) / kWarps;
    const int grid = (int)(need < resident ? need : resident);
    return launch_pdl(kernel, dim3(grid), dim3(kNormWarpThreads), smem, st, (const T *)y, (const T *)z, w, (T *)out,
                      C, GS, n_groups, rows, eps);
}

// rows of at most kNormWarpMaxVec * 32 vectors
template <typename T>
static cudaError_t norm_warp_dispatch(const void *y, const void *z, const float *w, void *out, int T_rows, int C,
                                      int n_groups, float eps, cudaStream_t st) {
    const int nvec = C / n_groups / Vec16<T>::n;
    switch ((nvec + 31) / 32) {
        case 1: return norm_warp_launch<T, 1>(y, z, w, out, T_rows, C, n_groups, eps, st);
        case 2: return norm_warp_launch<T, 2>(y, z, w, out, T_rows, C, n_groups, eps, st);
        case 3: return norm_warp_launch<T, 3>(y, z, w, out, T_rows, C, n_groups, eps, st);
        case 4: return norm_warp_launch<T, 4>(y, z, w, out, T_rows, C, n_groups, eps, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t norm_stream_launch(const void *y, const void *z, const float *w, void *out, int T_rows, int C,
                                      int n_groups, float eps, cudaStream_t st) {
    constexpr auto kernel = gated_rmsnorm_stream_kernel<T>;
    const int GS = C / n_groups;
    const int threads = (GS / kNormStreamElems + (GS % kNormStreamElems ? 1 : 0) + 31) / 32 * 32;
    const int smem = 2 * 2 * GS * (int)sizeof(T);
    const int rows = T_rows * n_groups;  // below 2^30 (the dispatcher's rule), so r + gridDim.x fits
    cudaError_t e = raise_smem_limit<kernel>(2 * 2 * kNormStreamRowBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem)) != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const long long resident = (long long)sms * per_sm;
    const int grid = rows < resident ? rows : (int)resident;
    return launch_pdl(kernel, dim3(grid), dim3(threads), smem, st, (const T *)y, (const T *)z, w, (T *)out, C, GS,
                      n_groups, rows, eps);
}

template <typename T>
static cudaError_t norm_launch(const void *y, const void *z, const float *w, void *out, int T_rows, int C,
                               int n_groups, float eps, cudaStream_t st) {
    const int GS = C / n_groups;
    const int smem = GS * (int)sizeof(float);
    if (smem > 48 * 1024) {  // once per device, to the largest group supported
        cudaError_t e = raise_smem_limit<gated_rmsnorm_kernel<T>>(kNormMaxGroup * (int)sizeof(float));
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(gated_rmsnorm_kernel<T>, dim3(T_rows, n_groups), dim3(kNormThreads), smem, st,
                      (const T *)y, (const T *)z, w, (T *)out, C, GS, eps);
}

cudaError_t launch_gated_rmsnorm(int dtype, const void *y, const void *z, const float *w, void *out, int T_rows,
                                 int C, int n_groups, float eps, cudaStream_t st) {
    const int GS = C / n_groups;
    const bool few_rows = (long long)T_rows * n_groups < (1ll << 30);
    const int warp_row_bytes = kNormWarpMaxVec * 32 * 16;  // 1024 bf16 or 512 float32 channels
    if (dtype == SSD_DTYPE_BF16) {
        if (few_rows && GS * 2 <= warp_row_bytes)
            return norm_warp_dispatch<__nv_bfloat16>(y, z, w, out, T_rows, C, n_groups, eps, st);
        if (few_rows && GS * 2 <= kNormStreamRowBytes)
            return norm_stream_launch<__nv_bfloat16>(y, z, w, out, T_rows, C, n_groups, eps, st);
        return norm_launch<__nv_bfloat16>(y, z, w, out, T_rows, C, n_groups, eps, st);
    }
    if (few_rows && GS * 4 <= warp_row_bytes)
        return norm_warp_dispatch<float>(y, z, w, out, T_rows, C, n_groups, eps, st);
    if (few_rows && GS * 4 <= kNormStreamRowBytes)
        return norm_stream_launch<float>(y, z, w, out, T_rows, C, n_groups, eps, st);
    return norm_launch<float>(y, z, w, out, T_rows, C, n_groups, eps, st);
}

}  // namespace ssd
