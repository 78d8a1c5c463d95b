// chunk_scan_fused.cu -- third kernel of the fused tensor-core prefill (bf16 storage, P = 64,
// N = 128): the outputs of every block, with the inter-block state carried on chip.
//
// For token l of 128-token block k, head h (acs = in-block inclusive cumsum of dt*A):
//   y_l = sum_{s<=l, s in k} (C_l . B_s) exp(acs_l - acs_s) dt_s x_s + exp(acs_l) C_l h_{k-1}^T
//         + D x_l
//   h_k = exp(acs_last) h_{k-1} + sum_{s in k} dt_s exp(acs_last - acs_s) x_s (outer) B_s
// Source: blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §1.1 (decay mask L = tril(exp(segsum)), the
// state passed between chunks) and §1.2 (the intra-chunk einsum); steps a2, a3, a5 of the
// chunked SSD; the D skip is Mamba-2's.
//
// Each CTA walks its range of units (runs.cuh) forward: per unit (batch, head pair, block) the
// C and B tiles are loaded once and CB = C_k B_k^T is formed once for both heads; per item
// (unit, head):
//   O   = C_k h_{k-1}^T   from a bf16 [n][p] tile that the chain warps write from the state
//   S   : H += B_k^T (w x_k), w_s = dt_s exp(acs_last - acs_s), into the head's state in TMEM,
//         which the chain warps have already scaled by exp(acs_last): H becomes h_k
//   P~  = mask(CB * dt_s exp(acs_l - acs_s)) + D on the diagonal (CUDA cores -> TMEM)
//   Y   = P~ x_k
//   y_l = Y_l + exp(acs_l) O_l
// The state entering the first block of each run is the carry-in that run_pass left in the
// run's slot.  So no per-block state ever leaves the SM: the chain of blocks within a run is
// the TMEM accumulator itself.  S here is a single bf16 product (w x rounded once): the state
// only feeds the O term through a bf16 tile; h_final comes from the hi/lo run states.
//
// Decay factors are kept as acs2 = acs * log2(e) and ldt = log2(dt), and an exponent is
// always (acs2_l - acs2_s) + ldt_s: the cumsums are subtracted before log2(dt) is added, which
// would otherwise be lost to rounding once the cumsum is large.  Padded tokens past L have
// dt = 0 (ldt = -inf) and take the last real token's cumsum exactly.  P~ factors through
// 32 x 32 sub-blocks as in chunk_scan_tc.cu (two factors at most 1 below the diagonal; a
// diagonal sub-block factors through its middle token when its cumsum falls by at most 96 in
// base 2, else one by one).
//
// Warp roles (every wait bounded; a timeout is recorded in the status word):
//   warp 0       TMA producer: C/B tiles per unit
//   warp 1       MMA issuer (one lane): CB per unit; O, S, Y per item
//   warps 2..3   decay factors: warp 2 + hh forms ldt and acs2 of head hh's items (the strided dt
//                loads of its next item issued before the current one is processed)
//   warps 4..7   transform: w x into a bf16 tile (32 rows per warp)
//   warps 8..15  P~ (two 32-column sub-blocks of 32 rows per warp)
//   warps 16..19 chain: state -> bf16 h^T tile, state *= exp(acs_last) (TMEM lane quarter each)
//   warps 20..23 epilogue: y = Y + exp(acs) O into a staging tile, one TMA store per item
//   warp 24      TMA producer of the x tiles, into a ring of kXS
#include "common.cuh"
#include "launch.h"
#include "runs.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace ssd {

namespace csf {
constexpr int R = 128, P = 64, N = 128;
constexpr int kPrepWarp = 2, kXformWarp = 4, kPtWarp = 8, kChainWarp = 16, kEpiWarp = 20, kXWarp = 24;
constexpr int kXform = 4, kPt = 8, kChain = 4, kEpi = 4;
constexpr int kThreads = (kXWarp + 1) * 32;
constexpr int kXS = 3;  // x ring
constexpr int kRS = 4;  // ring of decay-factor rows
constexpr uint32_t kBox = R * 128;  // [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kOffC = 0;                    // C: 2 n-boxes
constexpr uint32_t kOffB = 2 * kBox;             // B: 2 n-boxes
constexpr uint32_t kOffX = 4 * kBox;             // x ring
constexpr uint32_t kOffWx = kOffX + kXS * kBox;  // w x tiles [2]
constexpr uint32_t kOffHt = kOffWx + 2 * kBox;   // h^T tiles [2]
constexpr uint32_t kOffOut = kOffHt + 2 * kBox;  // y staging
constexpr uint32_t kOffRows = kOffOut + kBox;    // [kRS] x {ldt[128], acs2[128]}
constexpr uint32_t kRowBytes = 2 * R * 4;
constexpr uint32_t kOffVb = kOffRows + kRS * kRowBytes;  // per-P~-warp column factors
constexpr uint32_t kOffBar = kOffVb + kPt * 32 * 4;
constexpr uint32_t kSmem = kOffBar + 512 + 1024;
// TMEM columns
constexpr uint32_t kColCB = 0, kColPt = 128, kColH = 256, kColY = 384, kColO = 448;
constexpr uint32_t kTmemCols = 512;
constexpr float kDiagFactorRange = 96.f;
constexpr int kEpiBar = 1;
}  // namespace csf

// The CTA's items in order: units first to last, heads 0 and 1 of each; the unit's (batch,
// block, head pair) are stepped without division.
struct FwdItems {
    int u, k, q, b, nk, NQ;
    __device__ __forceinline__ FwdItems(int u0, int nk_, int NQ_) : u(u0), nk(nk_), NQ(NQ_) {
        const int ch = u0 / nk;
        k = u0 - ch * nk;
        b = ch / NQ;
        q = ch - b * NQ;
    }
    __device__ __forceinline__ void next_unit() {
        ++u;
        if (++k == nk) {
            k = 0;
            if (++q == NQ) {
                q = 0;
                ++b;
            }
        }
    }
};

__global__ void __launch_bounds__(csf::kThreads, 1) chunk_scan_fused_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
    const __nv_bfloat16 *__restrict__ dt, const float *__restrict__ A_log, const float *__restrict__ dt_bias,
    float dt_min, float dt_max, const float *__restrict__ D, const float *__restrict__ slots,
    int *__restrict__ status, int L, int H, int G, RunLayout lay) {
    using namespace csf;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *ld_full = bars;                 // C/B tiles landed
    uint64_t *ld_empty = ld_full + 1;         // MMA commit after the unit's last S and O
    uint64_t *cb_full = ld_empty + 1;         // MMA commit after CB
    uint64_t *cb_empty = cb_full + 1;         // P~ warps done with the unit's CB
    uint64_t *x_full = cb_empty + 1;          // [kXS]
    uint64_t *x_empty = x_full + kXS;         // [kXS] MMA commit after Y
    uint64_t *rows_full = x_empty + kXS;      // [kRS] decay factors written
    uint64_t *rows_empty = rows_full + kRS;   // [kRS] every reader done
    uint64_t *wx_full = rows_empty + kRS;     // [2] transform wrote w x
    uint64_t *ch_full = wx_full + 2;          // [2] chain wrote h^T and scaled the state
    uint64_t *s_done = ch_full + 2;           // [2] MMA commit after O and S of an item
    uint64_t *pt_full = s_done + 2;           // [2] P~ written
    uint64_t *pt_empty = pt_full + 2;         // [2] MMA commit after Y
    uint64_t *acc_full = pt_empty + 2;        // MMA commit after Y (Y and O complete)
    uint64_t *acc_empty = acc_full + 1;       // epilogue read Y and O
    uint64_t *fin = acc_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u0 = lay.first(blockIdx.x), u1 = lay.first(blockIdx.x + 1);
    const int cnt = kPairHeads * (u1 - u0);
    if (cnt <= 0) return;
    const int nk = lay.nk, NQ = H / kPairHeads, hpg = H / G;

    if (tid == 0) {
        mbar_init(ld_full, 1);
        mbar_init(ld_empty, 1);
        mbar_init(cb_full, 1);
        mbar_init(cb_empty, kPt);
        for (int i = 0; i < kXS; ++i) {
            mbar_init(&x_full[i], 1);
            mbar_init(&x_empty[i], 1);
        }
        for (int i = 0; i < kRS; ++i) {
            mbar_init(&rows_full[i], 1);
            mbar_init(&rows_empty[i], kXform + kPt + kChain + kEpi);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&wx_full[i], kXform);
            mbar_init(&ch_full[i], kChain);
            mbar_init(&s_done[i], 1);
            mbar_init(&pt_full[i], kPt);
            mbar_init(&pt_empty[i], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpi);
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();  // the carry-ins come from the kernel before
    dt = after_wait(dt);
    A_log = after_wait(A_log);
    dt_bias = after_wait(dt_bias);
    D = after_wait(D);
    slots = after_wait(slots);
    status = after_wait(status);

    auto rows = [&](int j) { return reinterpret_cast<float *>(smem + kOffRows + (uint32_t)(j % kRS) * kRowBytes); };
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (mbar_test(bar, parity)) return true;
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, status)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            FwdItems it(u0, nk, NQ);
            for (int m = 0; m < u1 - u0; ++m, it.next_unit()) {
                const int g = (it.q * kPairHeads) / hpg;
                if (m > 0 && !wait(ld_empty, (m - 1) & 1)) break;
                mbar_arrive_expect_tx(ld_full, 4 * kBox);
                tma_load_3d(smem + kOffC, &tm_c, g * N, it.k * R, it.b, ld_full);
                tma_load_3d(smem + kOffC + kBox, &tm_c, g * N + 64, it.k * R, it.b, ld_full);
                tma_load_3d(smem + kOffB, &tm_b, g * N, it.k * R, it.b, ld_full);
                tma_load_3d(smem + kOffB + kBox, &tm_b, g * N + 64, it.k * R, it.b, ld_full);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_cb = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t id_kmn = idesc_bf16_f32(128, 64, false, true);  // K-major A, MN-major B
            constexpr uint32_t id_mnmn = idesc_bf16_f32(128, 64, true, true);  // both MN-major
            const uint64_t dc = desc_kmajor_sw128(smem_u32(smem + kOffC));
            const uint64_t db = desc_kmajor_sw128(smem_u32(smem + kOffB));
            const uint64_t dbt = desc_mnmajor_sw128(smem_u32(smem + kOffB), kBox);  // B^T, M = n
            bool ok = true;
            for (int m = 0; m < u1 - u0 && ok; ++m) {
                // CB = C B^T once the tiles are in and the P~ warps are done with the last CB
                if (!wait(ld_full, m & 1)) break;
                if (m > 0 && !wait(cb_empty, (m - 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < N / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tmem + kColCB, desc_add(dc, off), desc_add(db, off), id_cb, kk > 0 ? 1u : 0u);
                }
                mma_commit(cb_full);
                for (int hh = 0; hh < kPairHeads; ++hh) {
                    const int j = m * kPairHeads + hh, t = j & 1, s = j % kXS;
                    if (!wait(&wx_full[t], (j >> 1) & 1) || !wait(&ch_full[t], (j >> 1) & 1) ||
                        (j >= 1 && !wait(acc_empty, (j - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dh = desc_mnmajor_sw128(smem_u32(smem + kOffHt + t * kBox), kBox);
                    const uint64_t dw = desc_mnmajor_sw128(smem_u32(smem + kOffWx + t * kBox), kBox);
                    const uint64_t dx = desc_mnmajor_sw128(smem_u32(smem + kOffX + s * kBox), kBox);
#pragma unroll
                    for (int kk = 0; kk < N / 16; ++kk)  // O = C h^T (K = n)
                        mma_ss(tmem + kColO, desc_add(dc, (kk >> 2) * kBox + (kk & 3) * 32), desc_add(dh, kk * 2048),
                               id_kmn, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)  // H += B^T (w x) (K = tokens)
                        mma_ss(tmem + kColH + hh * 64, desc_add(dbt, kk * 2048), desc_add(dw, kk * 2048), id_mnmn, 1u);
                    mma_commit(&s_done[t]);
                    if (hh == kPairHeads - 1) mma_commit(ld_empty);  // last reads of this unit's C and B
                    if (!wait(&pt_full[t], (j >> 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)  // Y = P~ x
                        mma_ts(tmem + kColY, tmem + kColPt + t * 64 + kk * 8, desc_add(dx, kk * 2048), id_kmn,
                               kk > 0 ? 1u : 0u);
                    mma_commit(acc_full);
                    mma_commit(&x_empty[s]);
                    mma_commit(&pt_empty[t]);
                }
            }
            mma_commit(fin);
            mbar_wait(fin, 0, status);
        }
    } else if (warp < kXformWarp) {
        // ---------------------------------------------------------------- decay factors
        // warp 2 + hh serves head hh's items; lane i forms tokens 4i .. 4i+3 of the block.
        const int hh = warp - kPrepWarp;
        FwdItems it(u0, nk, NQ), ahead(u0, nk, NQ);
        auto load_raw = [&](const FwdItems &c, float (&r)[4]) {
            const int h = c.q * kPairHeads + hh, t0 = c.k * R + lane * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                r[i] = t0 + i < L ? __bfloat162float(dt[((size_t)c.b * L + t0 + i) * H + h]) : 0.f;
        };
        float r0[4];
        load_raw(ahead, r0);
        ahead.next_unit();
        for (int m = 0; m < u1 - u0; ++m, it.next_unit()) {
            const int j = m * kPairHeads + hh;
            const int h = it.q * kPairHeads + hh, t0 = it.k * R + lane * 4;
            float raw[4] = {r0[0], r0[1], r0[2], r0[3]};
            if (m + 1 < u1 - u0) {  // the next item's dt, in flight while this one is formed
                load_raw(ahead, r0);
                ahead.next_unit();
            }
            const float bias = dt_bias ? __ldg(dt_bias + h) : 0.f;
            const float A = -expf(__ldg(A_log + h));
            const bool ok = j < kRS || wait(&rows_empty[j % kRS], ((j / kRS) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            float d[4], run = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d[i] = t0 + i < L ? discretise_dt(raw[i], bias, dt_min, dt_max) : 0.f;
                run += d[i] * A;
            }
            float acc = warp_inclusive_sum(run) - run;
            float lg[4], a2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc += d[i] * A;
                a2[i] = acc * kLog2e;
                lg[i] = log2f(d[i]);
            }
            const int tl = L - 1 - it.k * R;  // a ragged block: padded slots take the last real cumsum
            if (tl < R - 1) {
                const float mine = (tl >> 2) == lane ? ((tl & 3) == 0 ? a2[0] : (tl & 3) == 1 ? a2[1]
                                                        : (tl & 3) == 2 ? a2[2] : a2[3]) : 0.f;
                const float last = __shfl_sync(0xffffffffu, mine, tl >> 2);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (lane * 4 + i > tl) a2[i] = last;
            }
            float *rw = rows(j);
            reinterpret_cast<float4 *>(rw)[lane] = make_float4(lg[0], lg[1], lg[2], lg[3]);
            reinterpret_cast<float4 *>(rw + R)[lane] = make_float4(a2[0], a2[1], a2[2], a2[3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&rows_full[j % kRS]);
        }
    } else if (warp < kPtWarp) {
        // ---------------------------------------------------------------- transform
        // w_s x_s into bf16, w_s = exp2((acs2_last - acs2_s) + ldt_s); rows [32 tw, 32 tw + 32)
        const int tw = warp - kXformWarp;
        for (int j = 0; j < cnt; ++j) {
            const int t = j & 1, s = j % kXS, r = j % kRS;
            bool ok = wait(&x_full[s], (j / kXS) & 1) && wait(&rows_full[r], (j / kRS) & 1);
            if (ok && j >= 2) ok = wait(&s_done[t], ((j >> 1) - 1) & 1);  // the w x tile is free
            if (!__all_sync(0xffffffffu, ok)) break;
            const float *ldt = rows(j), *acs2 = ldt + R;
            const int row0 = tw * 32;
            const float wl = ex2_approx((acs2[R - 1] - acs2[row0 + lane]) + ldt[row0 + lane]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&rows_empty[r]);
            const uint8_t *xt = smem + kOffX + s * kBox;
            uint8_t *wt = smem + kOffWx + t * kBox;
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {  // 32 rows x 8 chunks = 256 chunks over 32 lanes
                const int idx = qq * 32 + lane;
                const int rl = idx >> 3, chunk = idx & 7;
                const float w = __shfl_sync(0xffffffffu, wl, rl);
                const uint32_t off = sw128_offset(row0 + rl, chunk);
                const uint4 raw = *reinterpret_cast<const uint4 *>(xt + off);
                const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&in[i]));
                    o[i] = pack_bf16x2(f.x * w, f.y * w);
                }
                *reinterpret_cast<uint4 *>(wt + off) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&wx_full[t]);
        }
    } else if (warp < kChainWarp) {
        // ---------------------------------------------------------------- P~
        const int rq = warp & 3, pc = (warp - kPtWarp) >> 2;
        const int myrow = rq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(rq * 32) << 16;
        float *vb = reinterpret_cast<float *>(smem + kOffVb) + (warp - kPtWarp) * 32;
        {  // the sub-blocks above the diagonal stay zero in both P~ buffers
            uint32_t zero[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int bi = 0; bi < 2; ++bi) {
                    const int cb = bi == 0 ? pc : 3 - pc;
                    if (cb > rq) tmem_st16(tmem + lane_base + kColPt + t * 64 + cb * 16, zero);
                }
        }
        FwdItems it(u0, nk, NQ);
        for (int m = 0; m < u1 - u0; ++m, it.next_unit()) {
            if (!__all_sync(0xffffffffu, wait(cb_full, m & 1))) break;
            bool ok = true;
            for (int hh = 0; hh < kPairHeads; ++hh) {
                const int j = m * kPairHeads + hh, t = j & 1, r = j % kRS;
                const float d = D ? __ldg(D + it.q * kPairHeads + hh) : 0.f;
                ok = wait(&rows_full[r], (j / kRS) & 1);
                if (ok && j >= 2) ok = wait(&pt_empty[t], ((j >> 1) - 1) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float *ldt = rows(j), *acs2 = ldt + R;
                const float al = acs2[myrow];
                const uint32_t pt = tmem + lane_base + kColPt + t * 64;
#pragma unroll
                for (int bi = 0; bi < 2; ++bi) {
                    const int cb = bi == 0 ? pc : 3 - pc;
                    if (cb > rq) continue;  // warp-uniform
                    const bool diag = cb == rq;
                    const bool factored = !diag || acs2[cb * 32] - acs2[cb * 32 + 31] <= kDiagFactorRange;
                    // factored: P~_ls = CB_ls * 2^(acs2_l - ref) * 2^((ref - acs2_s) + ldt_s)
                    const float ref = diag ? acs2[cb * 32 + 15] : acs2[cb * 32 + 31];
                    const float uu = ex2_approx(al - ref);
                    if (factored) vb[lane] = ex2_approx((ref - acs2[cb * 32 + lane]) + ldt[cb * 32 + lane]);
                    __syncwarp();
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {  // 16 columns at a time
                        const int c0 = cb * 32 + hf * 16;
                        float v[16];
                        tmem_ld16(tmem + lane_base + kColCB + c0, v);
                        tmem_wait_ld();
                        if (factored) {
                            const float4 *v4 = reinterpret_cast<const float4 *>(vb + hf * 16);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 c = v4[i];
                                v[4 * i + 0] *= uu * c.x;
                                v[4 * i + 1] *= uu * c.y;
                                v[4 * i + 2] *= uu * c.z;
                                v[4 * i + 3] *= uu * c.w;
                            }
                        } else {
                            const float4 *a4 = reinterpret_cast<const float4 *>(acs2 + c0);
                            const float4 *l4 = reinterpret_cast<const float4 *>(ldt + c0);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 a = a4[i], l = l4[i];
                                v[4 * i + 0] *= ex2_approx((al - a.x) + l.x);
                                v[4 * i + 1] *= ex2_approx((al - a.y) + l.y);
                                v[4 * i + 2] *= ex2_approx((al - a.z) + l.z);
                                v[4 * i + 3] *= ex2_approx((al - a.w) + l.w);
                            }
                        }
                        if (diag) {  // causal mask and the D skip; a select, so what lies above is dropped
                            const int ld = myrow - c0;
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] = i < ld ? v[i] : (i == ld ? v[i] + d : 0.f);
                        }
                        uint32_t packed[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                        tmem_st8(pt + c0 / 2, packed);
                    }
                    __syncwarp();  // vb is rewritten by the next sub-block
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&pt_full[t]);
                    mbar_arrive(&rows_empty[r]);
                    if (hh == kPairHeads - 1) mbar_arrive(cb_empty);
                }
            }
            if (!ok) break;
        }
    } else if (warp < kEpiWarp) {
        // ---------------------------------------------------------------- chain
        // TMEM lanes 32 (warp % 4) .. + 31 are rows n of the two heads' states H^T [n][p].  Per
        // item (unit, head): the state entering the block (the run's carry-in at a run's first
        // block, else H as the previous block's S left it) goes out as the bf16 h^T tile of the
        // O product, and H is scaled by the block's decay exp(acs_last), so that the S product
        // accumulating onto it leaves the state after the block.
        const int quarter = warp & 3;
        const int n = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        FwdItems it(u0, nk, NQ);
        for (int m = 0; m < u1 - u0; ++m, it.next_unit()) {
            const bool run_start = m == 0 || it.k == 0;
            const int slot = run_start ? lay.slot(it.u, blockIdx.x) : 0;
            bool ok = true;
            for (int hh = 0; hh < kPairHeads; ++hh) {
                const int j = m * kPairHeads + hh, t = j & 1, r = j % kRS;
                ok = wait(&rows_full[r], (j / kRS) & 1);
                // O and S of this head's previous item are done: H holds its state, the tile is free
                if (ok && j >= 2) ok = wait(&s_done[t], ((j >> 1) - 1) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float a = ex2_approx(rows(j)[2 * R - 1]);  // exp(acs_last) of this block
                uint8_t *ht = smem + kOffHt + t * kBox;
                const uint32_t hcol = tmem + lane_base + kColH + hh * 64;
                const float4 *cin = reinterpret_cast<const float4 *>(
                    slots + ((size_t)slot * kPairHeads + hh) * P * N + (size_t)n * P);
#pragma unroll
                for (int qc = 0; qc < 4; ++qc) {  // 16 columns (two 16-byte chunks of the tile) at a time
                    float v[16];
                    if (run_start) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 f = cin[qc * 4 + i];
                            v[4 * i] = f.x;
                            v[4 * i + 1] = f.y;
                            v[4 * i + 2] = f.z;
                            v[4 * i + 3] = f.w;
                        }
                    } else {
                        tmem_ld16(hcol + qc * 16, v);
                        tmem_wait_ld();
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        *reinterpret_cast<uint4 *>(ht + sw128_offset(n, qc * 2 + c)) =
                            make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                       pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
                    uint32_t sc[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) sc[i] = __float_as_uint(v[i] * a);
                    tmem_st16(hcol + qc * 16, sc);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&ch_full[t]);
                    mbar_arrive(&rows_empty[r]);
                }
            }
            if (!ok) break;
        }
    } else if (warp == kXWarp) {
        // ---------------------------------------------------------------- x producer
        if (lane == 0) {
            FwdItems it(u0, nk, NQ);
            for (int m = 0; m < u1 - u0; ++m, it.next_unit()) {
                bool ok = true;
                for (int hh = 0; hh < kPairHeads && ok; ++hh) {
                    const int j = m * kPairHeads + hh, s = j % kXS;
                    ok = j < kXS || wait(&x_empty[s], ((j / kXS) - 1) & 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&x_full[s], kBox);
                    tma_load_3d(smem + kOffX + s * kBox, &tm_x, (it.q * kPairHeads + hh) * P, it.k * R, it.b,
                                &x_full[s]);
                }
                if (!ok) break;
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // thread = token row of the block: y = Y + exp(acs_l) O over its 64 columns, in two halves
        const int quarter = warp & 3;
        const int myrow = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool leader = warp == kEpiWarp && lane == 0;
        FwdItems it(u0, nk, NQ);
        bool ok = true;
        for (int m = 0; m < u1 - u0 && ok; ++m, it.next_unit()) {
            for (int hh = 0; hh < kPairHeads; ++hh) {
                const int j = m * kPairHeads + hh, r = j % kRS;
                ok = wait(&rows_full[r], (j / kRS) & 1) && wait(acc_full, j & 1);
                ok = __all_sync(0xffffffffu, ok);
                if (leader) bulk_wait_read();  // the staging tile is free once the last store read it
                if (!named_barrier_and(kEpiBar, kEpi * 32, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float scale = ex2_approx(rows(j)[R + myrow]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&rows_empty[r]);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {  // 16 columns (two 16-byte chunks of the row) at a time
                    float yv[16], ov[16];
                    tmem_ld16(tmem + lane_base + kColY + q4 * 16, yv);
                    tmem_ld16(tmem + lane_base + kColO + q4 * 16, ov);
                    tmem_wait_ld();
                    uint32_t o[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        o[i] = pack_bf16x2(fmaf(scale, ov[2 * i], yv[2 * i]), fmaf(scale, ov[2 * i + 1], yv[2 * i + 1]));
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        *reinterpret_cast<uint4 *>(smem + kOffOut + sw128_offset(myrow, q4 * 2 + c)) =
                            make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                fence_proxy_async_smem();
                named_barrier(kEpiBar, kEpi * 32);
                if (leader) {
                    tma_store_3d(&tm_y, smem + kOffOut, (it.q * kPairHeads + hh) * P, it.k * R, it.b);
                    bulk_commit();
                }
            }
        }
        if (leader) bulk_wait_all();
    }

    __syncthreads();
    if (*abort_flag && tid == 0) {
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
    }
    allow_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_free(tmem, kTmemCols);
}

bool prefill_fused_supported(int dtype, int P, int N, int H, int G) {
    return prefill_tc_supported(dtype, P, N) && H % G == 0 && (H / G) % kPairHeads == 0;
}

cudaError_t launch_chunk_scan_fused(const void *x, const void *Bm, const void *Cm, const void *dt, const float *A_log,
                                    const float *dt_bias, float dt_min, float dt_max, const float *D,
                                    const float *slots, void *y, int *status, int B, int L, int H, int G,
                                    int64_t x_row, int64_t bc_row, const RunLayout &lay, cudaStream_t st) {
    using namespace csf;
    CUtensorMap tm_x, tm_b, tm_c, tm_y;
    cudaError_t e = make_tmap_bf16_3d(&tm_x, x, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)x_row * 2,
                                      (uint64_t)L * x_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_b, Bm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_c, Cm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_y, y, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)H * P * 2,
                          (uint64_t)L * H * P * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = raise_smem_limit<chunk_scan_fused_kernel>((int)kSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(chunk_scan_fused_kernel, dim3(lay.grid), dim3(kThreads), kSmem, st, tm_x, tm_b, tm_c, tm_y,
                      (const __nv_bfloat16 *)dt, A_log, dt_bias, dt_min, dt_max, D, slots, status, L, H, G, lay);
}

}  // namespace ssd
