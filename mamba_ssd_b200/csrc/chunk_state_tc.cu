// chunk_state_tc.cu -- step a3 on the tcgen05 tensor cores (bf16 storage, P = 64, N = 128):
//
//   S_k[p][n] = sum_{s in block k} w_s x_s[p] B_s[n],   w_s = dt_s exp(acs_last - acs_s)
//
// stored transposed as S_k^T [N][P] (the layout of the accumulator: TMEM lane n, column p)
//
// for every 128-token block k (the M of one tcgen05 MMA; the tensor-core path blocks the
// sequence in 128 tokens whatever chunk the caller asked for -- the decomposition is exact,
// only rounding differs), computed transposed as one M=128 (n) x N=64 (p) x K=128 (s)
// product per (batch, block, head): A = B_k^T and the B operand X'' = diag(w) x_k, both read
// MN-major straight from 128-byte-swizzled tiles.  The fp32 block state feeds the float32
// state pass and finally h_final, whose tolerance (1e-3 relative to its RMS) is tighter than
// one bf16 rounding of w_s x_s (RMS relative error 2^-9/sqrt(3) = 1.1e-3).  So X'' is split
// into bf16 hi + lo parts (hi = bf16(v), lo = bf16(v - hi), |v - hi - lo| <= 2^-17 |v|).  The lo
// box sits one MN atom after the hi box, so [hi | lo] is a single N = 128 operand: 8 MMAs of
// K=16 (M128 N128) into a 128-column fp32 accumulator whose halves the epilogue adds -- each
// MMA reads the shared A operand once for both parts.
//
// Source: the per-chunk state that the blog walk-through of "Compiler-First State Space
// Duality and Portable O(1) Autoregressive Caching for Inference" (bqwf.cn) §1.1 says is
// passed between chunks (the decay-weighted B^T X of each chunk).
//
// The kernel also forms step a1 for the items it owns (the decay factors that the state pass
// and the scan read): dt = clip(softplus(dt_raw + dt_bias)), A = -exp(A_log), the in-block
// cumsum acs of dt*A, stored in log2 form as acs2 = acs*log2(e) and ldt = log2(dt), so that
// dt_s exp(acs_l - acs_s) = exp2((acs2_l - acs2_s) + ldt_s).  The difference of the cumsums is
// taken before log2(dt) is added: folded into one number, log2(dt) would be lost to rounding
// once |acs2| is large (a decay of many nats per token).  Source: the
// blog walk-through's §1.1 (discretisation, chunked cumulative decay) and §1.2 (the fused
// softplus -> clip -> exp chain); §4.1 (the decay in float32).  Tokens past the end of their
// sequence get dt = 0, so their decay is 1 and their weight exactly 0 (ldt = -inf): in a packed
// varlen batch the x and B rows after a sequence's end, which belong to the next sequence, drop
// out of its last block's state that way.
//
// Structure: persistent CTAs, one per SM, each owning a contiguous range of (sequence, block,
// head) items of an equal-length or a packed varlen batch (items.cuh; consecutive items share
// the block's B tile).  Warp-specialised:
//   warp 0       TMA producer: B tile per (batch, block, group); x tile per item into a ring
//                of kStages stages
//   warps 18..21 decay factors of an item into its stage and to global memory (warp 18 + s
//                serves the items of stage s)
//   warp 1       MMA issuer (one lane): 8 MMAs per item into one of two TMEM accumulators
//   warps 2..9   transform: scale rows by w into hi (in place) and lo
//   warps 10..17 epilogue: drain an accumulator; each 32-column half (4 warps) stages its
//                columns in its own swizzled shared-memory box and writes them out with its own
//                TMA store (S^T, [N][P], fp32)
// Every role runs its own loop and the roles meet only at mbarriers (full/empty per stage,
// per accumulator, per B tile), so the tensor core, the transform of the next item and the
// drain of the previous one overlap.
#include "common.cuh"
#include "items.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace ssd {

namespace cst {
constexpr int R = 128, P = 64, N = 128;
constexpr int kXform = 8, kEpi = 8;
constexpr int kPrepWarp = 2 + kXform + kEpi;  // first of kStages decay-factor warps
constexpr int kStages = 4;
constexpr int kThreads = (kPrepWarp + kStages) * 32;
constexpr uint32_t kBox = R * 128;                 // [128 rows][64 bf16], 16 KB
constexpr uint32_t kOffB = 0;                      // B block: 2 n-boxes, 32 KB
constexpr uint32_t kStageBytes = 2 * kBox + 1024;  // x/hi box, lo box, ldt[128] + acs2[128]
constexpr uint32_t kOffStage = 2 * kBox;
constexpr uint32_t kOffOut = kOffStage + kStages * kStageBytes;  // S^T staging: 2 x [128][32] fp32
constexpr uint32_t kOffBar = kOffOut + 2 * kBox;
constexpr int kEpiBar = 1;  // named barriers of the epilogue's two column halves: 1 and 2
constexpr uint32_t kSmem = kOffBar + 256 + 1024;  // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 256;               // two 128-column fp32 accumulators [hi | lo]
}  // namespace cst

template <bool VARLEN>
__global__ void __launch_bounds__(cst::kThreads, 1) chunk_state_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_s, const __nv_bfloat16 *__restrict__ dt, const float *__restrict__ A_log,
    const float *__restrict__ dt_bias, float dt_min, float dt_max, float *__restrict__ dtf,
    float *__restrict__ acs, int *__restrict__ status, int reset_status, int L, int H, int G, int nk, int total,
    const Varlen vl) {
    using namespace cst;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *st_full = bars;                 // [kStages] TMA + decay factors -> transform
    uint64_t *op_full = st_full + kStages;    // [kStages] transform -> MMA (operands written)
    uint64_t *st_empty = op_full + kStages;   // [kStages] MMA commit -> producer
    uint64_t *acc_full = st_empty + kStages;  // [2] MMA commit -> epilogue
    uint64_t *acc_empty = acc_full + 2;       // [2] epilogue -> MMA
    uint64_t *b_full = acc_empty + 2;         // B tile landed
    uint64_t *b_empty = b_full + 1;           // MMA commit after the last item of a tile
    uint64_t *fin = b_empty + 1;              // MMA commit after the last MMA of the CTA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int first = (int)((long long)blockIdx.x * total / gridDim.x);
    const int cnt = (int)((long long)(blockIdx.x + 1) * total / gridDim.x) - first;
    if (cnt <= 0) return;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&st_full[i], 2);  // the producer's expect_tx arrive + the prep warp
            mbar_init(&op_full[i], kXform);
            mbar_init(&st_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kEpi);
        }
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_s);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // prologue done: from here on global memory is touched, after the previous kernel
    grid_dependency_wait();
    dt = after_wait(dt);
    A_log = after_wait(A_log);
    dt_bias = after_wait(dt_bias);
    dtf = after_wait(dtf);
    acs = after_wait(acs);
    status = after_wait(status);
    const Varlen tab = {after_wait(vl.tok0), after_wait(vl.blk0), after_wait(vl.seq), vl.n};
    // this call's status word starts clean (a later wait of the call may record a timeout),
    // unless the caller keeps one word across several calls (the varlen prefill)
    if (reset_status && blockIdx.x == 0 && tid == 0) *status = SSD_OK;

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
            // x is read once here: marked first to leave L2, so that the block states written
            // meanwhile stay there for the state pass
            const uint64_t stream_policy = l2_evict_first();
            ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
            int tiles = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int h = it.h();
                if (j == 0 || it.tile_first()) {
                    if (tiles > 0 && !wait(b_empty, (tiles - 1) & 1)) break;
                    mbar_arrive_expect_tx(b_full, 2 * kBox);
                    tma_load_3d(smem + kOffB, &tm_b, it.g * N, it.row(), it.zb, b_full);
                    tma_load_3d(smem + kOffB + kBox, &tm_b, it.g * N + 64, it.row(), it.zb, b_full);
                    ++tiles;
                }
                const int s = j % kStages;
                if (j >= kStages && !wait(&st_empty[s], ((j / kStages) - 1) & 1)) break;
                uint8_t *st = stage(j);
                mbar_arrive_expect_tx(&st_full[s], kBox);
                tma_load_3d_hint(st, &tm_x, h * P, it.row(), it.zb, &st_full[s], stream_policy);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true, true);  // N = [hi | lo]
            const uint64_t da = desc_mnmajor_sw128(smem_u32(smem + kOffB), kBox);
            ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
            int tiles = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int s = j % kStages, a = j & 1;
                if (j == 0 || it.tile_first()) {
                    if (!wait(b_full, tiles & 1)) break;
                    ++tiles;
                }
                if (!wait(&op_full[s], (j / kStages) & 1)) break;
                if (j >= 2 && !wait(&acc_empty[a], ((j >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint64_t dh = desc_mnmajor_sw128(smem_u32(stage(j)), kBox);  // [hi | lo] at LBO kBox
                const uint32_t d = tmem + (uint32_t)(a * 128);
#pragma unroll
                for (int kk = 0; kk < R / 16; ++kk)
                    mma_ss(d, desc_add(da, kk * 2048), desc_add(dh, kk * 2048), idesc, kk > 0 ? 1u : 0u);
                mma_commit(&acc_full[a]);
                mma_commit(&st_empty[s]);
                if (j == cnt - 1 || it.tile_last()) mma_commit(b_empty);
            }
            // every MMA (and every arrive it triggers) has landed before TMEM is released
            mma_commit(fin);
            mbar_wait(fin, 0, status);
        }
    } else if (warp >= kPrepWarp) {
        // ---------------------------------------------------------------- decay factors
        // warp kPrepWarp + s serves the items j = s, s + kStages, ... (those of stage s).  Lane
        // i: tokens 4i .. 4i+3 of the block (the same per-lane order and warp scan as the
        // stand-alone decay kernel, so both give the same bits).  The strided dt loads of the
        // next item are issued before this one is processed.
        const int s = warp - kPrepWarp;
        auto load_raw = [&](const ItemCursor<VARLEN> &c, float (&r)[4]) {
            const int t0 = c.k * R + lane * 4, h = c.h();  // t0: token of the sequence
            const size_t row = (size_t)c.zb * L + c.row0 + t0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                r[i] = t0 + i < c.len ? __bfloat162float(dt[(row + i) * H + h]) : 0.f;
        };
        auto step = [&](ItemCursor<VARLEN> &c) {
#pragma unroll
            for (int i = 0; i < kStages; ++i) c.next();
        };
        auto load_par = [&](const ItemCursor<VARLEN> &c, float &bias, float &alog) {
            bias = dt_bias ? __ldg(dt_bias + c.h()) : 0.f;
            alog = __ldg(A_log + c.h());
        };
        ItemCursor<VARLEN> it(first + s, H, G, nk, L, tab), ahead(first + s, H, G, nk, L, tab);
        float r0[4] = {0.f, 0.f, 0.f, 0.f}, b0 = 0.f, l0 = 0.f;
        if (s < cnt) {
            load_raw(ahead, r0);
            load_par(ahead, b0, l0);
        }
        step(ahead);
        for (int j = s; j < cnt; j += kStages) {
            float r1[4] = {0.f, 0.f, 0.f, 0.f}, b1 = 0.f, l1 = 0.f;
            if (j + kStages < cnt) {
                load_raw(ahead, r1);
                load_par(ahead, b1, l1);
            }
            const int h = it.h(), t0 = it.k * R + lane * 4;
            const float bias = b0;
            const float A = -expf(l0);
            bool ok = j < kStages || wait(&st_empty[s], ((j / kStages) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            float d[4], run = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d[i] = t0 + i < it.len ? discretise_dt(r0[i], bias, dt_min, dt_max) : 0.f;
                run += d[i] * A;
            }
            float acc = warp_inclusive_sum(run) - run;  // exclusive prefix of this lane
            float lg[4], a2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc += d[i] * A;
                a2[i] = acc * kLog2e;
                lg[i] = log2f(d[i]);
            }
            // a ragged last block: the padded slots take exactly the last real token's cumsum
            // (the lanes' partial sums round differently; the block's end must stand for that
            // token, so that its own weight exp2(acs2_end - acs2_last) is exactly 1)
            const int tl = it.len - 1 - it.k * R;  // slot of the last real token
            if (tl < R - 1) {                 // warp-uniform
                const float mine = (tl >> 2) == lane ? ((tl & 3) == 0 ? a2[0] : (tl & 3) == 1 ? a2[1]
                                                        : (tl & 3) == 2 ? a2[2] : a2[3]) : 0.f;
                const float last = __shfl_sync(0xffffffffu, mine, tl >> 2);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (lane * 4 + i > tl) a2[i] = last;
            }
            const float4 c4 = make_float4(lg[0], lg[1], lg[2], lg[3]);
            const float4 a4 = make_float4(a2[0], a2[1], a2[2], a2[3]);
            float *rows = reinterpret_cast<float *>(stage(j) + 2 * kBox);
            reinterpret_cast<float4 *>(rows)[lane] = c4;
            reinterpret_cast<float4 *>(rows + R)[lane] = a4;
            const size_t g = ((size_t)h * (total / H) + it.gblk()) * R + (size_t)lane * 4;  // head-major rows
            *reinterpret_cast<float4 *>(dtf + g) = c4;
            *reinterpret_cast<float4 *>(acs + g) = a4;
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_full[s]);
#pragma unroll
            for (int i = 0; i < 4; ++i) r0[i] = r1[i];
            b0 = b1;
            l0 = l1;
            step(it);
            step(ahead);
        }
    } else if (warp < 2 + kXform) {
        // ---------------------------------------------------------------- transform
        const int tw = warp - 2;  // rows [16 tw, 16 tw + 16)
        for (int j = 0; j < cnt; ++j) {
            const int s = j % kStages;
            if (!__all_sync(0xffffffffu, wait(&st_full[s], (j / kStages) & 1))) break;  // warp-uniform
            uint8_t *xt = stage(j);
            uint8_t *lo = xt + kBox;
            const float *ldt = reinterpret_cast<const float *>(xt + 2 * kBox);
            const float *acs2 = ldt + R;
            // w_s = dt_s exp(acs_last - acs_s) = exp2((acs2_last - acs2_s) + ldt_s); lanes 0..15
            // hold the weights of this warp's 16 rows
            const int rw = tw * 16 + (lane & 15);
            const float wl = lane < 16 ? ex2_approx((acs2[R - 1] - acs2[rw]) + ldt[rw]) : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 16 rows x 8 chunks = 128 chunks over 32 lanes
                const int idx = q * 32 + lane;
                const int rl = idx >> 3, chunk = idx & 7;
                const int row = tw * 16 + rl;
                const float w = __shfl_sync(0xffffffffu, wl, rl);
                const uint32_t off = sw128_offset(row, chunk);
                uint4 raw = *reinterpret_cast<const uint4 *>(xt + off);
                uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t hi[4], lw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&in[i]));
                    const float a0 = f.x * w, a1 = f.y * w;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
                    const float2 hf = __bfloat1622float2(h2);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                    hi[i] = *reinterpret_cast<const uint32_t *>(&h2);
                    lw[i] = *reinterpret_cast<const uint32_t *>(&l2);
                }
                *reinterpret_cast<uint4 *>(xt + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&op_full[s]);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // TMEM lane quarter (warp % 4) = rows n, column half = p range of 32
        // The two column halves (4 warps each, one TMEM lane quarter per warp) drain, stage and
        // store their own 32-column box independently: each half has its own named barrier and
        // its own TMA store, so neither waits for the other.
        const int quarter = warp & 3, half = (warp - 2 - kXform) >> 2;
        const int n = quarter * 32 + lane;
        const bool leader = ((warp - 2 - kXform) & 3) == 0 && lane == 0;  // issues this half's stores
        const int bar = kEpiBar + half;
        // the block states stay in L2 for the state pass, which reads them next and then drops
        // their lines (they are never needed in DRAM)
        const uint64_t keep = l2_evict_last();
        uint8_t *box = smem + kOffOut + half * kBox;
        ItemCursor<VARLEN> it(first, H, G, nk, L, tab);
        for (int j = 0; j < cnt; ++j, it.next()) {
            const int a = j & 1;
            const bool ok = __all_sync(0xffffffffu, wait(&acc_full[a], (j >> 1) & 1));
            float v[32];
            if (ok) {
                tc_fence_after();
                // columns [0, 64) hold the hi part's products, [64, 128) the lo part's
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 128 + half * 32);
                float w[32];
                tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_ld16(taddr + 64, *reinterpret_cast<float(*)[16]>(&w[0]));
                tmem_ld16(taddr + 80, *reinterpret_cast<float(*)[16]>(&w[16]));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] += w[i];
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[a]);
            }
            // the staging tile is free once the previous item's stores have read it
            if (leader) bulk_wait_read();
            if (!named_barrier_and(bar, kEpi / 2 * 32, ok)) break;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<float4 *>(box + sw128_offset(n, c)) =
                    make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_proxy_async_smem();
            named_barrier(bar, kEpi / 2 * 32);
            if (leader) {
                const int row = (int)(((size_t)it.gblk() * H + it.h()) * N);
                tma_store_2d_hint(&tm_s, box, half * 32, row, keep);
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

bool prefill_tc_supported(int dtype, int P, int N) {
    return dtype == SSD_DTYPE_BF16 && P == cst::P && N == cst::N;
}

cudaError_t launch_chunk_state_tc(const void *x, const void *Bm, const void *dt, const float *A_log,
                                  const float *dt_bias, float dt_min, float dt_max, float *dtf, float *acs,
                                  float *states, int *status, bool reset_status, int B, int L, int H, int G,
                                  int64_t x_row, int64_t bc_row, const Varlen &vl, int nblocks, int num_sms,
                                  cudaStream_t st) {
    using namespace cst;
    const int nk = cdiv(L, R);  // blocks per sequence of an equal-length batch
    const int total = nblocks * H;
    CUtensorMap tm_x, tm_b, tm_s;
    // x and B rows are x_row and bc_row elements apart (H*P and G*N when dense)
    cudaError_t e = make_tmap_bf16_3d(&tm_x, x, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)x_row * 2,
                                      (uint64_t)L * x_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_b, Bm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    // S^T of every item as rows of 64 fp32: TMA boxes of 32 columns x 128 rows
    e = make_tmap_f32_2d(&tm_s, states, (uint64_t)P, (uint64_t)total * N, (uint64_t)P * 4, 32, R);
    if (e != cudaSuccess) return e;
    const int grid = total < num_sms ? total : num_sms;
    auto launch = [&](auto tag) {
        constexpr auto kernel = decltype(tag)::kernel;
        cudaError_t r = raise_smem_limit<kernel>((int)kSmem);
        if (r != cudaSuccess) return r;
        return launch_pdl(kernel, dim3(grid), dim3(kThreads), kSmem, st, tm_x, tm_b, tm_s, (const __nv_bfloat16 *)dt,
                          A_log, dt_bias, dt_min, dt_max, dtf, acs, status, reset_status ? 1 : 0, L, H, G, nk, total, vl);
    };
    return vl.n ? launch(KernelTag<chunk_state_tc_kernel<true>>{}) : launch(KernelTag<chunk_state_tc_kernel<false>>{});
}

}  // namespace ssd
