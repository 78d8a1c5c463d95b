// chunk_scan_tc.cu -- steps a2 + a5 on the tcgen05 tensor cores (bf16 storage, P = 64,
// N = 128): the intra-block masked product, the carried-in state and the D skip.
//
// For token l of 128-token block k, head h (acs = in-block cumsum of dt*A):
//   y_l = sum_{s<=l, s in k} (C_l . B_s) exp(acs_l - acs_s) dt_s x_s + exp(acs_l) C_l h_prev^T
//         + D x_l
// Source: blog walk-through of "Compiler-First State Space Duality and Portable O(1)
// Autoregressive Caching for Inference" (bqwf.cn) §1.1 (decay mask L = tril(exp(segsum)),
// state passed between chunks) and §1.2 (the intra-chunk einsum); the D skip is Mamba-2's.
//
// The sequence is blocked in 128 tokens, the M of one tcgen05 MMA (the blog's 256 is the
// TPU v6e MXU size; the decomposition is exact for any block size).  Per item (batch,
// block, head):
//   CB  = C_k B_k^T                 once per (batch, block, group), kept in TMEM, fp32
//   O   = C_k h_prev^T              h_prev^T arrives by TMA as a bf16 [n][p] tile
//   P~  = mask(CB * dt_s * exp(acs_l - acs_s)) + D on the diagonal   (CUDA cores -> TMEM,
//         from precomputed per-token factors acs2 = acs*log2(e) and ldt = log2(dt); the
//         exponent is (acs2_l - acs2_s) + ldt_s, the cumsums subtracted first so that ldt is
//         not lost to rounding when the cumsum is large)
//   Y   = P~ x_k                    A operand read from TMEM, x_k straight from its TMA tile
//   y_l = Y_l + exp(acs_l) O_l      (epilogue, fp32 -> bf16)
// Folding dt into the columns of P~ and D into its diagonal means x is used as loaded:
// no x operand is rewritten, and no x is re-read for the skip.
//
// The decay factor of P~ is formed per 32 x 32 sub-block.  Below the diagonal (rows in
// sub-block r, columns in sub-block c < r) it factors through the cumsum at the last token
// of column sub-block c:
//   dt_s exp(acs_l - acs_s) = exp(acs_l - acs_ref) * dt_s exp(acs_ref - acs_s),
// both factors at most 1 since acs is non-increasing, so a 32 x 32 sub-block costs 64
// exponentials instead of 1024.  A diagonal sub-block factors through its middle token when
// the cumsum falls by at most 96 (base 2) across it, so neither factor leaves fp32's range;
// otherwise its factors are taken one by one.  Above the diagonal P~ is zero: those TMEM
// columns are cleared once per CTA and never written again.
//
// Structure: persistent CTAs own contiguous ranges of items ordered (sequence, block, head) of
// an equal-length or a packed varlen batch (items.cuh), so consecutive items share the C/B
// tiles and CB.  Warp-specialised, every role with its own
// loop, the roles meeting only at mbarriers:
//   warp 0       TMA producer: C/B tiles per (batch, block, group); x tile, h_prev^T tile and
//                the item's per-token factors into a ring of kStages stages
//   warp 1       MMA issuer (one lane): CB per tile; O and Y per item into one of two TMEM sets
//   warps 2..9   P~ of an item into its TMEM set
//   warps 10..17 epilogue: y = Y + exp(acs) O of an item; each 32-column half (4 warps) stages
//                its columns in its own swizzled shared-memory box that its own TMA store
//                writes out (tokens past L are clipped by the store); the
//                ragged last block of a packed varlen sequence is stored row by row instead,
//                its real rows only, since the rows after it belong to the next sequence
//                (their P~ rows only ever meet x rows after the sequence's end through the
//                causal mask's zeros, so they cannot reach a real row)
// so the tensor core runs item j's products while P~ of item j+1 is formed and item j-1's
// outputs are written.
#include "common.cuh"
#include "items.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace ssd {

namespace csc {
constexpr int R = 128, P = 64, N = 128;
constexpr int kPt = 8, kEpi = 8;
constexpr int kThreads = (2 + kPt + kEpi) * 32;
constexpr int kStages = 4;
constexpr uint32_t kBox = R * 128;            // [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kOffC = 0;                 // C block: 2 n-boxes, 32 KB
constexpr uint32_t kOffB = 2 * kBox;          // B block: 2 n-boxes, 32 KB
constexpr uint32_t kOffStage = 4 * kBox;      // ring of stages
constexpr uint32_t kStX = 0, kStH = kBox, kStRows = 2 * kBox;  // x box, h_prev^T box, ldt+acs2
constexpr uint32_t kStageBytes = 2 * kBox + 2048;             // keeps 1024-byte alignment
constexpr uint32_t kOffOut = kOffStage + kStages * kStageBytes;  // y staging [128][64] bf16
constexpr uint32_t kOffVb = kOffOut + kBox;                       // per-warp column factors
constexpr uint32_t kOffBar = kOffVb + kPt * 32 * 4;
constexpr uint32_t kSmem = kOffBar + 256 + 1024;
// TMEM columns: CB, then two sets of {P~ (bf16 pairs), Y, O}
constexpr uint32_t kColCB = 0, kSet = 192, kSet0 = 128, kOffPT = 0, kOffY = 64, kOffO = 128;
constexpr uint32_t kTmemCols = 512;
constexpr float kDiagFactorRange = 96.f;  // log2 range of a diagonal sub-block that is factored
constexpr int kEpiBar = 1;                 // named barriers of the epilogue's two column halves: 1, 2
}  // namespace csc

template <bool VARLEN>
__global__ void __launch_bounds__(csc::kThreads, 1) chunk_scan_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_h,
    const __grid_constant__ CUtensorMap tm_y, const float *__restrict__ dtf, const float *__restrict__ acs,
    const float *__restrict__ D, __nv_bfloat16 *__restrict__ y, const __nv_bfloat16 *__restrict__ hT,
    int *__restrict__ status, int L, int H, int G, int nk, int total, const Varlen vl) {
    using namespace csc;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *st_full = bars;                  // [kStages] TMA -> P~, MMA
    uint64_t *st_empty = st_full + kStages;    // [kStages] MMA commit after Y -> producer
    uint64_t *ld_full = st_empty + kStages;    // C/B tiles landed
    uint64_t *ld_empty = ld_full + 1;          // MMA commit after the last O of a tile
    uint64_t *cb_full = ld_empty + 1;          // MMA commit after CB
    uint64_t *cb_empty = cb_full + 1;          // P~ warps done reading CB of a tile
    uint64_t *pt_full = cb_empty + 1;          // [2] P~ warps wrote P~ of a set
    uint64_t *acc_full = pt_full + 2;          // [2] MMA commit after Y
    uint64_t *acc_empty = acc_full + 2;        // [2] epilogue read Y, O of a set
    uint64_t *fin = acc_empty + 2;             // MMA commit after the last MMA of the CTA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int first = (int)((long long)blockIdx.x * total / gridDim.x);
    const int cnt = (int)((long long)(blockIdx.x + 1) * total / gridDim.x) - first;
    if (cnt <= 0) return;
    const int nblk = total / H;  // blocks of the whole batch

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&st_full[i], 1);
            mbar_init(&st_empty[i], 1);
        }
        mbar_init(ld_full, 1);
        mbar_init(ld_empty, 1);
        mbar_init(cb_full, 1);
        mbar_init(cb_empty, kPt);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pt_full[i], kPt);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kEpi);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_h);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // prologue done: from here on global memory is touched, after the previous kernel
    grid_dependency_wait();
    dtf = after_wait(dtf);
    acs = after_wait(acs);
    D = after_wait(D);
    y = after_wait(y);
    hT = after_wait(hT);
    status = after_wait(status);
    const Varlen tab = {after_wait(vl.tok0), after_wait(vl.blk0), after_wait(vl.seq), vl.n};

    auto stage = [&](int j) { return smem + kOffStage + (uint32_t)(j % kStages) * kStageBytes; };
    // a bounded wait that gives up at once when another role has already timed out
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
            const uint64_t release = l2_evict_first();  // x and h_prev^T: their last read, first to leave L2
            ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
            int tiles = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int h = it.h();
                if (j == 0 || it.tile_first()) {
                    if (tiles > 0 && !wait(ld_empty, (tiles - 1) & 1)) break;
                    mbar_arrive_expect_tx(ld_full, 4 * kBox);
                    tma_load_3d(smem + kOffC, &tm_c, it.g * N, it.row(), it.zb, ld_full);
                    tma_load_3d(smem + kOffC + kBox, &tm_c, it.g * N + 64, it.row(), it.zb, ld_full);
                    tma_load_3d(smem + kOffB, &tm_b, it.g * N, it.row(), it.zb, ld_full);
                    tma_load_3d(smem + kOffB + kBox, &tm_b, it.g * N + 64, it.row(), it.zb, ld_full);
                    ++tiles;
                }
                const int s = j % kStages;
                if (j >= kStages && !wait(&st_empty[s], ((j / kStages) - 1) & 1)) break;
                uint8_t *st = stage(j);
                const size_t row = ((size_t)h * nblk + it.gblk()) * R;  // head-major factor rows
                mbar_arrive_expect_tx(&st_full[s], 2 * kBox + 2 * R * 4);
                tma_load_3d_hint(st + kStX, &tm_x, h * P, it.row(), it.zb, &st_full[s], release);
                tma_load_2d_hint(st + kStH, &tm_h, 0, (int)(((size_t)it.gblk() * H + h) * N), &st_full[s], release);
                bulk_load(st + kStRows, dtf + row, R * 4, &st_full[s]);
                bulk_load(st + kStRows + R * 4, acs + row, R * 4, &st_full[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_cb = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t id_kmn = idesc_bf16_f32(128, 64, false, true);  // K-major A, MN-major B
            const uint64_t dc = desc_kmajor_sw128(smem_u32(smem + kOffC));
            const uint64_t db = desc_kmajor_sw128(smem_u32(smem + kOffB));
            ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
            int tiles = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int s = j % kStages, t = j & 1;
                const uint32_t set = tmem + kSet0 + t * kSet;
                if (j == 0 || it.tile_first()) {  // CB = C B^T, once P~ is done with the previous CB
                    if (!wait(ld_full, tiles & 1)) break;
                    if (tiles > 0 && !wait(cb_empty, (tiles - 1) & 1)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < N / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                        mma_ss(tmem + kColCB, desc_add(dc, off), desc_add(db, off), id_cb, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(cb_full);
                    ++tiles;
                }
                if (!wait(&st_full[s], (j / kStages) & 1)) break;
                if (j >= 2 && !wait(&acc_empty[t], ((j >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint64_t dh = desc_mnmajor_sw128(smem_u32(stage(j) + kStH), kBox);
                const uint64_t dx = desc_mnmajor_sw128(smem_u32(stage(j) + kStX), kBox);
#pragma unroll
                for (int kk = 0; kk < N / 16; ++kk)  // O = C h_prev^T
                    mma_ss(set + kOffO, desc_add(dc, (kk >> 2) * kBox + (kk & 3) * 32), desc_add(dh, kk * 2048),
                           id_kmn, kk > 0 ? 1u : 0u);
                if (!wait(&pt_full[t], (j >> 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < R / 16; ++kk)  // Y = P~ x
                    mma_ts(set + kOffY, set + kOffPT + kk * 8, desc_add(dx, kk * 2048), id_kmn, kk > 0 ? 1u : 0u);
                mma_commit(&acc_full[t]);
                mma_commit(&st_empty[s]);
                if (j == cnt - 1 || it.tile_last()) mma_commit(ld_empty);
            }
            // every MMA (and every arrive it triggers) has landed before TMEM is released
            mma_commit(fin);
            mbar_wait(fin, 0, status);
        }
    } else if (warp < 2 + kPt) {
        // ---------------------------------------------------------------- P~
        // TMEM lanes 32 (warp % 4) .. + 31 are rows rq of the block; this warp forms the
        // 32-column sub-blocks pc and 3 - pc of those rows (those above the diagonal are zero)
        const int rq = warp & 3, pc = (warp - 2) >> 2;
        const int myrow = rq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(rq * 32) << 16;
        float *vb = reinterpret_cast<float *>(smem + kOffVb) + (warp - 2) * 32;
        {
            uint32_t zero[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int bi = 0; bi < 2; ++bi) {
                    const int cb = bi == 0 ? pc : 3 - pc;
                    if (cb > rq) tmem_st16(tmem + lane_base + kSet0 + t * kSet + kOffPT + cb * 16, zero);
                }
        }
        ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
        int tiles = 0;
        for (int j = 0; j < cnt; ++j, it.next()) {
            const int s = j % kStages, t = j & 1;
            const float d = D ? __ldg(D + it.h()) : 0.f;  // issued before the waits
            if (j == 0 || it.tile_first()) {
                if (!__all_sync(0xffffffffu, wait(cb_full, tiles & 1))) break;
                ++tiles;
            }
            bool ok = wait(&st_full[s], (j / kStages) & 1);
            // P~ of this set was last read by the MMA of item j - 2
            if (ok && j >= 2) ok = wait(&acc_full[t], ((j >> 1) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform
            tc_fence_after();
            const float *ldt = reinterpret_cast<const float *>(stage(j) + kStRows);
            const float *acs2 = ldt + R;
            const float al = acs2[myrow];
            const uint32_t set = tmem + lane_base + kSet0 + t * kSet;
#pragma unroll
            for (int bi = 0; bi < 2; ++bi) {
                const int cb = bi == 0 ? pc : 3 - pc;
                if (cb > rq) continue;  // warp-uniform
                const bool diag = cb == rq;
                const bool factored = !diag || acs2[cb * 32] - acs2[cb * 32 + 31] <= kDiagFactorRange;
                if (!factored) {
                    // a diagonal sub-block whose decay spans more than fp32 can factor: each factor on
                    // its own, 16 columns at a time (rare: only steep in-block decay takes it)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int c0 = cb * 32 + hf * 16;
                        float v[16];
                        tmem_ld16(tmem + lane_base + kColCB + c0, v);
                        tmem_wait_ld();
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
                        const int ld = myrow - c0;  // causal mask and the D skip, by select
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = i < ld ? v[i] : (i == ld ? v[i] + d : 0.f);
                        uint32_t packed[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) packed[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                        tmem_st8(set + kOffPT + c0 / 2, packed);
                    }
                    continue;
                }
                float v[32];
                tmem_ld16(tmem + lane_base + kColCB + cb * 32, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(tmem + lane_base + kColCB + cb * 32 + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
                {
                    // P~_ls = CB_ls * 2^(acs2_l - ref) * 2^((ref - acs2_s) + ldt_s)
                    const float ref = diag ? acs2[cb * 32 + 15] : acs2[cb * 32 + 31];
                    vb[lane] = ex2_approx((ref - acs2[cb * 32 + lane]) + ldt[cb * 32 + lane]);
                    __syncwarp();
                    const float u = ex2_approx(al - ref);
                    tmem_wait_ld();
                    const float4 *v4 = reinterpret_cast<const float4 *>(vb);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 c = v4[i];
                        v[4 * i + 0] *= u * c.x;
                        v[4 * i + 1] *= u * c.y;
                        v[4 * i + 2] *= u * c.z;
                        v[4 * i + 3] *= u * c.w;
                    }
                    __syncwarp();
                }
                if (diag) {  // causal mask and the D skip; a select, so what lies above is dropped
                    const int ld = myrow - cb * 32;
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = i < ld ? v[i] : (i == ld ? v[i] + d : 0.f);
                }
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                tmem_st16(set + kOffPT + cb * 16, packed);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&pt_full[t]);
                if (j == cnt - 1 || it.tile_last()) mbar_arrive(cb_empty);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int rq = warp & 3, half = (warp - 2 - kPt) >> 2;  // TMEM lane quarter, 32 columns
        const int myrow = rq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(rq * 32) << 16;
        // The two column halves (4 warps each, one TMEM lane quarter per warp) stage and store
        // their own 32-column box (64-byte rows, 64-byte swizzle) with their own named barrier
        // and TMA store, so neither waits for the other.
        const bool leader = ((warp - 2 - kPt) & 3) == 0 && lane == 0;  // issues this half's stores
        const int bar = kEpiBar + half;
        uint8_t *box = smem + kOffOut + half * (kBox / 2);
        ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
        for (int j = 0; j < cnt; ++j, it.next()) {
            const int t = j & 1, h = it.h();
            // exp(acs_l) from the log2-form cumsum; read here, the stage may be refilled by now
            const float al = __ldg(acs + ((size_t)h * nblk + it.gblk()) * R + myrow);
            // a packed sequence's ragged last block: the rows after its end belong to the next
            // sequence, so its real rows are stored directly instead of by the tile store
            const int direct = VARLEN ? it.valid() : R;
            const bool ok = __all_sync(0xffffffffu, wait(&acc_full[t], (j >> 1) & 1));
            uint32_t o[16];
            if (ok) {
                tc_fence_after();
                const uint32_t set = tmem + lane_base + kSet0 + t * kSet;
                float yv[32], ov[32];
                tmem_ld16(set + kOffY + half * 32, *reinterpret_cast<float(*)[16]>(&yv[0]));
                tmem_ld16(set + kOffY + half * 32 + 16, *reinterpret_cast<float(*)[16]>(&yv[16]));
                tmem_ld16(set + kOffO + half * 32, *reinterpret_cast<float(*)[16]>(&ov[0]));
                tmem_ld16(set + kOffO + half * 32 + 16, *reinterpret_cast<float(*)[16]>(&ov[16]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[t]);
                // the item's h_prev^T tile (128 rows of 128 bytes) was read by its TMA load, which
                // completed before the MMA that produced O: it is dead, and its lines leave L2
                // without a write-back (only this item reads them)
                if (half == 0) discard_l2_line(hT + ((size_t)it.gblk() * H + h) * N * P + (size_t)myrow * P);
                const float scale = ex2_approx(al);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    o[i] = pack_bf16x2(fmaf(scale, ov[2 * i], yv[2 * i]), fmaf(scale, ov[2 * i + 1], yv[2 * i + 1]));
            }
            // the staging tile is free once the previous item's store has read it
            if (leader) bulk_wait_read();
            if (!named_barrier_and(bar, kEpi / 2 * 32, ok)) break;
            if (direct < R) {  // item-uniform
                if (myrow < direct) {
                    uint4 *dst = reinterpret_cast<uint4 *>(y + ((size_t)it.row() + myrow) * H * P + (size_t)h * P +
                                                           half * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                }
                continue;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4 *>(box + sw64_offset(myrow, q)) =
                    make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            fence_proxy_async_smem();
            named_barrier(bar, kEpi / 2 * 32);
            if (leader) {
                tma_store_3d(&tm_y, box, h * P + half * 32, it.row(), it.zb);
                bulk_commit();
            }
        }
        if (leader) bulk_wait_all();
    }

    __syncthreads();
    if (*abort_flag && tid == 0) {
        // a wait timed out: let copies still in flight land (bounded) before the CTA exits
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
    }
    allow_dependents();  // this CTA's work is done: the next kernel may take its SM
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_free(tmem, kTmemCols);
}

cudaError_t launch_chunk_scan_tc(const void *x, const void *Bm, const void *Cm, const float *dtf,
                                 const float *acs, const __nv_bfloat16 *hT, const float *D, void *y,
                                 int *status, int B, int L, int H, int G, int64_t x_row, int64_t bc_row,
                                 const Varlen &vl, int nblocks, int num_sms, cudaStream_t st) {
    using namespace csc;
    const int nk = cdiv(L, R);  // blocks per sequence of an equal-length batch
    const int total = nblocks * H;
    CUtensorMap tm_x, tm_b, tm_c, tm_h, tm_y;
    // x, B and C rows are x_row and bc_row elements apart (H*P and G*N when dense); y is dense
    cudaError_t e = make_tmap_bf16_3d(&tm_x, x, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)x_row * 2,
                                      (uint64_t)L * x_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_b, Bm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_c, Cm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_2d(&tm_h, hT, (uint64_t)P, (uint64_t)nblocks * H * N, (uint64_t)P * 2, 64, R);
    if (e != cudaSuccess) return e;
    // y leaves in 32-column boxes, one per epilogue half
    e = make_tmap_bf16_3d_sw64(&tm_y, y, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)H * P * 2,
                               (uint64_t)L * H * P * 2, 32, R, 1);
    if (e != cudaSuccess) return e;
    const int grid = total < num_sms ? total : num_sms;
    auto launch = [&](auto tag) {
        constexpr auto kernel = decltype(tag)::kernel;
        cudaError_t r = raise_smem_limit<kernel>((int)kSmem);
        if (r != cudaSuccess) return r;
        return launch_pdl(kernel, dim3(grid), dim3(kThreads), kSmem, st, tm_x, tm_b, tm_c, tm_h, tm_y, dtf, acs, D,
                          (__nv_bfloat16 *)y, hT, status, L, H, G, nk, total, vl);
    };
    return vl.n ? launch(KernelTag<chunk_scan_tc_kernel<true>>{}) : launch(KernelTag<chunk_scan_tc_kernel<false>>{});
}

}  // namespace ssd
