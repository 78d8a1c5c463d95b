// chunk_scan_tc.cu -- steps a2 + a5 on the tcgen05 tensor cores (bf16 storage, P = 64,
// N = 128, chunk 256): the intra-chunk masked product, the carried-in state and the D skip.
//
// For token l of chunk c, head h (acs = in-chunk cumsum of dt*A, X' = dt x):
//   y_l = sum_{s<=l, s in c} (C_l . B_s) exp(acs_l - acs_s) X'_s + exp(acs_l) C_l h_prev^T + D x_l
// Source: blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §1.1 (decay mask L = tril(exp(segsum)),
// state passed between chunks) and §1.2 (the intra-chunk einsum); the D skip is Mamba-2's.
//
// The 256-token chunk is processed as two 128-row halves, the M of one tcgen05 MMA.  The
// lower-left 128 x 128 block of the mask factorises exactly through the state after token
// 127 of the chunk, h_mid = exp(acs_127) h_prev + S_0 with S_0 = sum_{s<128}
// exp(acs_127 - acs_s) X'_s (outer) B_s, so for the second half
//   y_l = [masked diagonal block] + exp(acs_l - acs_127) C_l h_mid^T + D x_l,
// and no exponential outside the two diagonal blocks is ever taken (both factors of the
// split are <= 1: nothing overflows).  Per item (batch, 128-row half, head):
//   half 0: CB = C_0 B_0^T,  Y = P~ X'_0,  O = C_0 h_prev^T
//   half 1: CB = C_1 B_1^T,  S_0^T = B_0^T X~_0,  Y = P~ X'_1,  O = C_1 h_mid^T
// where P~ = mask(CB * exp(acs_l - acs_s)) is formed on the CUDA cores from CB read out of
// TMEM and written back to TMEM as bf16, and consumed from there as the A operand (the
// ".kind::f16 [d], [a-tmem], b-desc" form); all other operands come from 128-byte-swizzled
// shared-memory tiles written by TMA or by the CUDA cores.  Accumulation is fp32 in TMEM.
//
// Persistent CTAs own contiguous ranges of items ordered (batch, half-chunk, head), so
// consecutive items share the C/B tiles and the CB product of their (batch, half, group);
// the next item's x tile is prefetched by TMA while the current one computes.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace ssd {

namespace csc {
constexpr int Q = 256, R = 128, P = 64, N = 128;
constexpr int kThreads = 256;  // 8 warps: two per TMEM lane quarter
constexpr uint32_t kBox = R * 128;      // one [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kOffC = 0;           // C half: 2 n-boxes                              32 KB
constexpr uint32_t kOffB = 32768;       // B rows 0..127 (2 boxes), rows 128..255 (2)      64 KB
constexpr uint32_t kOffX0 = 98304;      // x stage 0: rows 0..127 box, rows 128..255 box    32 KB
constexpr uint32_t kOffX1 = 131072;     // x stage 1                                         32 KB
constexpr uint32_t kOffH = 163840;      // h_prev^T or h_mid^T, [n][p] bf16 MN-major         16 KB
constexpr uint32_t kOffHp = 180224;     // h_prev slab [p][n] fp32 (bulk copy)               32 KB
constexpr uint32_t kOffRows = 212992;   // per stage: dt[256], acs[256]                       2 x 2 KB
constexpr uint32_t kRowBytes = 2 * Q * 4;
constexpr uint32_t kOffBar = kOffRows + 2 * kRowBytes;
constexpr uint32_t kSmem = kOffBar + 128 + 1024;
// TMEM columns
constexpr uint32_t kColCB = 0, kColPT = 128, kColY = 192, kColO = 256, kColS = 320;
constexpr uint32_t kTmemCols = 512;
}  // namespace csc

__global__ void __launch_bounds__(csc::kThreads, 1) chunk_scan_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const __nv_bfloat16 *__restrict__ x,
    const float *__restrict__ dtf, const float *__restrict__ acs, const float *__restrict__ hprev,
    const float *__restrict__ D, __nv_bfloat16 *__restrict__ y, int *__restrict__ status, int L,
    int H, int G, int nc, int nsub, int total) {
    using namespace csc;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *bar_ld = bars + 0;   // C/B tiles
    uint64_t *bar_x = bars + 1;    // [2] x stages (+ dt/acs rows)
    uint64_t *bar_cb = bars + 3;   // CB product
    uint64_t *bar_s0 = bars + 4;   // S_0 product (and O of half 0)
    uint64_t *bar_y = bars + 5;    // Y product
    uint64_t *bar_o = bars + 6;    // O product of half 1
    uint64_t *bar_hp = bars + 7;   // h_prev slab
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
    const float *hps = reinterpret_cast<const float *>(smem + kOffHp);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 (rows of the half) and split columns
    const int rq = warp & 3, ch = warp >> 2;
    const int myrow = rq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(rq * 32) << 16;
    const int first = (int)((long long)blockIdx.x * total / gridDim.x);
    const int cnt = (int)((long long)(blockIdx.x + 1) * total / gridDim.x) - first;
    if (cnt <= 0) return;
    const int hpg = H / G;
    const size_t Lp = (size_t)nc * Q;

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_c);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // item -> (b, sub-chunk sc, head h); chunk c = sc / 2, half = sc % 2
    auto decode = [&](int j, int &b, int &sc, int &h) {
        const int it = first + j;
        h = it % H;
        const int t = it / H;
        sc = t % nsub;
        b = t / nsub;
    };
    auto tile_key = [&](int j) {
        int b, sc, h;
        decode(j, b, sc, h);
        return (b * nsub + sc) * G + h / hpg;
    };
    // thread 0: x rows of the chunk up to this half (S_0 needs rows 0..127) + dt/acs rows
    auto issue_x = [&](int j) {
        int b, sc, h;
        decode(j, b, sc, h);
        const int c = sc >> 1, half = sc & 1, s = j & 1;
        uint8_t *dst = smem + (s ? kOffX1 : kOffX0);
        uint8_t *rows = smem + kOffRows + s * kRowBytes;
        const size_t row = ((size_t)b * H + h) * Lp + (size_t)c * Q;
        mbar_arrive_expect_tx(&bar_x[s], (half + 1) * kBox + kRowBytes);
        tma_load_3d(dst, &tm_x, h * P, c * Q, b, &bar_x[s]);
        if (half) tma_load_3d(dst + kBox, &tm_x, h * P, c * Q + R, b, &bar_x[s]);
        bulk_load(rows, dtf + row, Q * 4, &bar_x[s]);
        bulk_load(rows + Q * 4, acs + row, Q * 4, &bar_x[s]);
    };
    auto issue_hp = [&](int j) {  // thread 0: the h_prev slab [P][N] fp32 of item j
        int b, sc, h;
        decode(j, b, sc, h);
        const int c = sc >> 1;
        mbar_arrive_expect_tx(bar_hp, P * N * 4);
        bulk_load(smem + kOffHp, hprev + (((size_t)b * nc + c) * H + h) * (size_t)(P * N), P * N * 4, bar_hp);
    };
    auto issue_tiles = [&](int j) {  // thread 0: C rows of this half, B rows 0..half*128+127
        int b, sc, h;
        decode(j, b, sc, h);
        const int c = sc >> 1, half = sc & 1, g = h / hpg;
        const int row = c * Q + half * R;
        mbar_arrive_expect_tx(bar_ld, (2 + 2 * (half + 1)) * kBox);
        tma_load_3d(smem + kOffC, &tm_c, g * N, row, b, bar_ld);
        tma_load_3d(smem + kOffC + kBox, &tm_c, g * N + 64, row, b, bar_ld);
        for (int hh = 0; hh <= half; ++hh) {
            tma_load_3d(smem + kOffB + hh * 2 * kBox, &tm_b, g * N, c * Q + hh * R, b, bar_ld);
            tma_load_3d(smem + kOffB + hh * 2 * kBox + kBox, &tm_b, g * N + 64, c * Q + hh * R, b, bar_ld);
        }
    };

    int ld_issued = 0, ld_done = 0, x_issued[2] = {0, 0}, x_done[2] = {0, 0};
    int cb_issued = 0, cb_done = 0, s0_issued = 0, s0_done = 0, y_issued = 0, y_done = 0;
    int o_issued = 0, o_done = 0, hp_issued = 0, hp_done = 0;
    bool ok = true;

    constexpr uint32_t id_cb = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t id_kmn = idesc_bf16_f32(128, 64, false, true);  // K-major A, MN-major B
    constexpr uint32_t id_mnmn = idesc_bf16_f32(128, 64, true, true);

    if (tid == 0) {
        issue_x(0);
        issue_hp(0);
    }
    x_issued[0] = 1;
    hp_issued = 1;

    // scale the rows [row0, row0 + 128) of a swizzled x box in place by w(row)
    auto scale_box = [&](uint8_t *box, auto wfun) {
#pragma unroll 4
        for (int q = tid; q < R * 8; q += kThreads) {
            const int row = q >> 3, chunk = q & 7;
            const uint32_t off = sw128_offset(row, chunk);
            const float w = wfun(row);
            uint4 raw = *reinterpret_cast<const uint4 *>(box + off);
            uint32_t *u = reinterpret_cast<uint32_t *>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[i]));
                u[i] = pack_bf16x2(f.x * w, f.y * w);
            }
            *reinterpret_cast<uint4 *>(box + off) = raw;
        }
    };
    // row n = myrow of the MN-major h^T tile, columns p in [32 ch, 32 ch + 32)
    auto store_hT = [&](const float (&v)[P / 2]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint4 w = make_uint4(pack_bf16x2(v[k * 8 + 0], v[k * 8 + 1]), pack_bf16x2(v[k * 8 + 2], v[k * 8 + 3]),
                                 pack_bf16x2(v[k * 8 + 4], v[k * 8 + 5]), pack_bf16x2(v[k * 8 + 6], v[k * 8 + 7]));
            *reinterpret_cast<uint4 *>(smem + kOffH + sw128_offset(myrow, ch * 4 + k)) = w;
        }
    };

    for (int j = 0; j < cnt; ++j) {
        const int s = j & 1;
        int b, sc, h;
        decode(j, b, sc, h);
        const int c = sc >> 1, half = sc & 1;
        // prefetch the next item's x and rows (its stage was last used by item j-1, complete)
        if (j + 1 < cnt) {
            if (tid == 0) issue_x(j + 1);
            ++x_issued[s ^ 1];
        }
        // C/B tiles and the CB product when (batch, half-chunk, group) changes
        if (j == 0 || tile_key(j) != tile_key(j - 1)) {
            if (tid == 0) issue_tiles(j);
            ++ld_issued;
            ok = mbar_wait_all(bar_ld, ld_done & 1, status);
            if (!ok) break;
            ++ld_done;
            if (tid == 0) {
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + kOffC);
                const uint32_t b0 = smem_u32(smem + kOffB + half * 2 * kBox);
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
                    mma_ss(tmem + kColCB, desc_kmajor_sw128(a0 + off), desc_kmajor_sw128(b0 + off), id_cb,
                           k > 0 ? 1u : 0u);
                }
                mma_commit(bar_cb);
            }
            ++cb_issued;
        }
        ok = mbar_wait_all(&bar_x[s], x_done[s] & 1, status);
        if (!ok) break;
        ++x_done[s];
        const float *dts = reinterpret_cast<const float *>(smem + kOffRows + s * kRowBytes);
        const float *acsr = dts + Q;

        // X' = dt x for this half's rows and, for half 1, X~_0 = dt exp(acs_127 - acs) x on
        // rows 0..127, both in place in the stage buffer
        uint8_t *xs = smem + (s ? kOffX1 : kOffX0);
        scale_box(xs + half * kBox, [&](int r) { return dts[half * R + r]; });
        if (half) {
            const float a127 = acsr[R - 1];
            scale_box(xs, [&](int r) { return dts[r] * __expf(a127 - acsr[r]); });
        }
        ok = mbar_wait_all(bar_hp, hp_done & 1, status);  // h_prev slab of this item
        if (!ok) break;
        ++hp_done;
        if (!half) {  // h_prev^T tile for O = C_0 h_prev^T; the slab is free afterwards
            float v[P / 2];
#pragma unroll
            for (int p = 0; p < P / 2; ++p) v[p] = hps[(ch * 32 + p) * N + myrow];
            store_hT(v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            if (!half) {  // O = C_0 h_prev^T
                const uint32_t a0 = smem_u32(smem + kOffC), hb = smem_u32(smem + kOffH);
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k)
                    mma_ss(tmem + kColO, desc_kmajor_sw128(a0 + (k >> 2) * kBox + (k & 3) * 32),
                           desc_mnmajor_sw128(hb + k * 2048, kBox), id_kmn, k > 0 ? 1u : 0u);
                if (j + 1 < cnt) issue_hp(j + 1);
            } else {  // S_0^T = B_0^T X~_0
                const uint32_t b0 = smem_u32(smem + kOffB), xt = smem_u32(xs);
#pragma unroll 1
                for (int k = 0; k < R / 16; ++k)
                    mma_ss(tmem + kColS, desc_mnmajor_sw128(b0 + k * 2048, kBox), desc_mnmajor_sw128(xt + k * 2048, kBox),
                           id_mnmn, k > 0 ? 1u : 0u);
            }
            mma_commit(bar_s0);
        }
        ++s0_issued;
        if (!half && j + 1 < cnt) ++hp_issued;

        // P~ = mask(CB * exp(acs_l - acs_s)) -> TMEM as bf16 (row l = lane of this thread)
        if (cb_done < cb_issued) {
            ok = mbar_wait_all(bar_cb, cb_done & 1, status);
            if (!ok) break;
            ++cb_done;
        }
        tc_fence_after();
        {
            const int l = myrow;  // row inside the half
            const float al = acsr[half * R + l] * kLog2e;
#pragma unroll 1
            for (int blk = ch; blk < 4; blk += 2) {  // the two warps of a lane quarter split the blocks
                uint32_t packed[16];
                if (blk > rq) {  // entirely above the diagonal for these rows
#pragma unroll
                    for (int i = 0; i < 16; ++i) packed[i] = 0u;
                } else {
                    float v0[16], v1[16];
                    tmem_ld16(tmem + lane_base + kColCB + blk * 32, v0);
                    tmem_ld16(tmem + lane_base + kColCB + blk * 32 + 16, v1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int sa = blk * 32 + 2 * i, sb = sa + 1;
                        const float ca = i < 8 ? v0[2 * i] : v1[2 * i - 16];
                        const float cb = i < 8 ? v0[2 * i + 1] : v1[2 * i + 1 - 16];
                        const float pa = sa <= l ? ca * exp2f(al - acsr[half * R + sa] * kLog2e) : 0.f;
                        const float pb = sb <= l ? cb * exp2f(al - acsr[half * R + sb] * kLog2e) : 0.f;
                        packed[i] = pack_bf16x2(pa, pb);
                    }
                }
                tmem_st16(tmem + lane_base + kColPT + blk * 16, packed);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // Y = P~ X'_half
            tc_fence_after();
            const uint32_t xb = smem_u32(xs + half * kBox);
#pragma unroll 1
            for (int k = 0; k < R / 16; ++k)
                mma_ts(tmem + kColY, tmem + kColPT + k * 8, desc_mnmajor_sw128(xb + k * 2048, kBox), id_kmn,
                       k > 0 ? 1u : 0u);
            mma_commit(bar_y);
        }
        ++y_issued;

        // half 1: h_mid = exp(acs_127) h_prev + S_0 -> h^T, then O = C_1 h_mid^T
        ok = mbar_wait_all(bar_s0, s0_done & 1, status);
        if (!ok) break;
        ++s0_done;
        if (half) {
            tc_fence_after();
            const float a127 = __expf(acsr[R - 1]);
            float v[P / 2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float sv[16];
                tmem_ld16(tmem + lane_base + kColS + ch * 32 + q * 16, sv);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[q * 16 + i] = fmaf(a127, hps[(ch * 32 + q * 16 + i) * N + myrow], sv[i]);
            }
            store_hT(v);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + kOffC), hb = smem_u32(smem + kOffH);
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k)
                    mma_ss(tmem + kColO, desc_kmajor_sw128(a0 + (k >> 2) * kBox + (k & 3) * 32),
                           desc_mnmajor_sw128(hb + k * 2048, kBox), id_kmn, k > 0 ? 1u : 0u);
                mma_commit(bar_o);
                if (j + 1 < cnt) issue_hp(j + 1);  // the slab was read above, before the sync
            }
            ++o_issued;
            if (j + 1 < cnt) ++hp_issued;
        }

        // epilogue: y = Y + scale * O + D x, scale = exp(acs_l) or exp(acs_l - acs_127).
        // The x row is fetched into registers before waiting for the products.
        const int l = myrow;
        const int tok = c * Q + half * R + l;
        const bool live = tok < L;
        const size_t rowoff = (((size_t)b * L + (live ? tok : 0)) * H + h) * P + ch * 32;
        uint4 xr[4];
        if (live) {
#pragma unroll
            for (int k = 0; k < 4; ++k) xr[k] = __ldg(reinterpret_cast<const uint4 *>(x + rowoff) + k);
        }
        if (half) {
            ok = mbar_wait_all(bar_o, o_done & 1, status);
            if (!ok) break;
            ++o_done;
        }
        ok = mbar_wait_all(bar_y, y_done & 1, status);
        if (!ok) break;
        ++y_done;
        tc_fence_after();
        {
            const float scale = __expf(acsr[half * R + l] - (half ? acsr[R - 1] : 0.f));
            const float d = D ? D[h] : 0.f;
            uint4 *yr = reinterpret_cast<uint4 *>(y + rowoff);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float t0[16], t1[16];
                tmem_ld16(tmem + lane_base + kColY + ch * 32 + q * 16, t0);
                tmem_ld16(tmem + lane_base + kColO + ch * 32 + q * 16, t1);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int k = q * 2 + cc;
                        uint32_t *u = reinterpret_cast<uint32_t *>(&xr[k]);
                        uint32_t o[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[i]));
                            const int e = cc * 8 + 2 * i;
                            o[i] = pack_bf16x2(fmaf(scale, t1[e], t0[e]) + d * f.x,
                                               fmaf(scale, t1[e + 1], t0[e + 1]) + d * f.y);
                        }
                        yr[k] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (!ok) {
        // a wait timed out: drain whatever is still in flight (bounded) before releasing TMEM
        while (ld_done < ld_issued && mbar_wait(bar_ld, ld_done & 1, nullptr)) ++ld_done;
        for (int s = 0; s < 2; ++s)
            while (x_done[s] < x_issued[s] && mbar_wait(&bar_x[s], x_done[s] & 1, nullptr)) ++x_done[s];
        while (hp_done < hp_issued && mbar_wait(bar_hp, hp_done & 1, nullptr)) ++hp_done;
        while (cb_done < cb_issued && mbar_wait(bar_cb, cb_done & 1, nullptr)) ++cb_done;
        while (s0_done < s0_issued && mbar_wait(bar_s0, s0_done & 1, nullptr)) ++s0_done;
        while (y_done < y_issued && mbar_wait(bar_y, y_done & 1, nullptr)) ++y_done;
        while (o_done < o_issued && mbar_wait(bar_o, o_done & 1, nullptr)) ++o_done;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_free(tmem, kTmemCols);
}

bool chunk_scan_tc_supported(int dtype, int P, int N, int chunk) {
    return dtype == SSD_DTYPE_BF16 && P == csc::P && N == csc::N && chunk == csc::Q;
}

cudaError_t launch_chunk_scan_tc(const void *x, const void *Bm, const void *Cm, const float *dtf,
                                 const float *acs, const float *hprev, const float *D, void *y,
                                 int *status, int B, int L, int H, int G, int num_sms, cudaStream_t st) {
    using namespace csc;
    const int nc = cdiv(L, Q), nsub = cdiv(L, R);
    const int total = B * nsub * H;
    CUtensorMap tm_x, tm_b, tm_c;
    cudaError_t e = make_tmap_bf16_3d(&tm_x, x, (uint64_t)H * P, (uint64_t)L, (uint64_t)B,
                                      (uint64_t)H * P * 2, (uint64_t)L * H * P * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_b, Bm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)G * N * 2,
                          (uint64_t)L * G * N * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_c, Cm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)G * N * 2,
                          (uint64_t)L * G * N * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    const int grid = total < num_sms ? total : num_sms;
    cudaFuncSetAttribute(chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    chunk_scan_tc_kernel<<<grid, kThreads, kSmem, st>>>(tm_x, tm_b, tm_c, (const __nv_bfloat16 *)x, dtf, acs,
                                                        hprev, D, (__nv_bfloat16 *)y, status, L, H, G, nc,
                                                        nsub, total);
    return cudaGetLastError();
}

}  // namespace ssd
