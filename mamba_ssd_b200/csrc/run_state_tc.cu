// run_state_tc.cu -- first kernel of the fused tensor-core prefill (bf16 storage, P = 64,
// N = 128): the state each run of blocks leaves behind when it starts from zero,
//
//   S_run[p][n] = sum_{s in run} dt_s exp(sum_{t = s+1 .. end of run} dA_t) x_s[p] B_s[n]
//
// and the run's total decay, log2 of exp(sum_{t in run} dA_t), for each of the two heads of
// the run's head pair (runs and slots: runs.cuh).  That is the chunk-state step of the
// chunked SSD (step a3) taken over a whole run at once: the state passed between chunks
// (blog walk-through of "Compiler-First State Space Duality and Portable O(1) Autoregressive
// Caching for Inference", bqwf.cn, §1.1) is linear, so the states of the run's blocks,
// chained through the blocks' decays, are one sum whose weights decay from each token to the
// run's end.  The kernel also forms step a1 for its tokens (dt = clip(softplus(dt_raw +
// dt_bias)), dA = dt * -exp(A_log), blog §1.1, §1.2, §4.1, in float32).
//
// The blocks of a run are walked from its last block to its first, so the weight exponent
// of token s -- the suffix sum of dA after s within the run -- is the in-block suffix sum
// plus the decay of the blocks already done; the run's last real token gets exactly
// exp2(0) = 1 times its dt (the padded tokens past L have dA = 0 and add exact zeros).
//
// The product is one accumulation chain per (run, head) in TMEM: per block, M=128 (n) x N=128
// ([hi | lo] of w x, p) x K=128 (s), A = B^T and B = the scaled x, both MN-major from
// 128-byte-swizzled tiles; the accumulate flag is off for the run's first block.  The scaled
// x is split into bf16 hi + lo parts (|w x - hi - lo| <= 2^-17 |w x|) because the run state
// feeds h_final, whose tolerance (1e-3 relative to its RMS) is tighter than one bf16
// rounding.  The epilogue adds the halves and stores S_run^T ([N][P], the accumulator's
// layout) to the run's slot.
//
// Structure: persistent CTAs over the unit ranges of runs.cuh, warp-specialised, the roles
// meeting only at mbarriers (every wait bounded; a timeout is recorded in the status word):
//   warp 0       TMA producer: B tile per unit into one of two slots; x tile per item into a
//                ring of kStages stages
//   warp 1       MMA issuer (one lane): 8 MMAs per item into the (run parity, head) accumulator
//   warps 2..3   decay factors: warp 2 + hh serves head hh's items in order, carrying the
//                decay of the run's later blocks; writes log2 of each token's weight into the
//                stage and the run's decay to the workspace
//   warps 4..11  transform: w x into bf16 hi (in place) and lo
//   warps 12..19 epilogue: drain a run's accumulator through a swizzled staging tile and two
//                TMA stores
#include "common.cuh"
#include "launch.h"
#include "runs.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace ssd {

namespace rst {
constexpr int R = 128, P = 64, N = 128;
constexpr int kPrep = 2, kXform = 8, kEpi = 8;
constexpr int kXformWarp = 2 + kPrep, kEpiWarp = kXformWarp + kXform;
constexpr int kThreads = (kEpiWarp + kEpi) * 32;
constexpr int kStages = 3;
constexpr uint32_t kBox = R * 128;                 // [128 rows][64 bf16], 16 KB
constexpr uint32_t kOffB = 0;                      // two B tiles of 2 n-boxes each, 64 KB
constexpr uint32_t kStageBytes = 2 * kBox + 1024;  // x/hi box, lo box, lw[128] (+ pad)
constexpr uint32_t kOffStage = 4 * kBox;
constexpr uint32_t kOffOut = kOffStage + kStages * kStageBytes;  // S^T staging: 2 x [128][32] fp32
constexpr uint32_t kOffBar = kOffOut + 2 * kBox;
constexpr int kEpiBar = 1;
constexpr uint32_t kSmem = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;  // four 128-column accumulators: (run parity, head)
}  // namespace rst

// The CTA's items in this kernel's order: runs in order, the blocks of a run from last to
// first, heads 0 and 1 of the pair for each block.
struct RevItems {
    int u1, nk;
    int rs, re, u, hh, r;  // current run [rs, re), unit, head, run index within the CTA
    __device__ __forceinline__ RevItems(int u0, int u1_, int nk_) : u1(u1_), nk(nk_), rs(u0), hh(0), r(0) {
        re = min(u1, (u0 / nk + 1) * nk);
        u = re - 1;
    }
    __device__ __forceinline__ bool run_first() const { return u == re - 1; }  // first block processed
    __device__ __forceinline__ bool run_last() const { return u == rs; }       // last block processed
    __device__ __forceinline__ void next() {
        if (++hh < kPairHeads) return;
        hh = 0;
        if (u > rs) {
            --u;
            return;
        }
        rs = re;
        re = min(u1, (rs / nk + 1) * nk);
        u = re - 1;
        ++r;
    }
};

__global__ void __launch_bounds__(rst::kThreads, 1) run_state_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_s, const __nv_bfloat16 *__restrict__ dt, const float *__restrict__ A_log,
    const float *__restrict__ dt_bias, float dt_min, float dt_max, float *__restrict__ decay_out,
    int *__restrict__ status, int reset_status, int L, int H, int G, RunLayout lay) {
    using namespace rst;
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *st_full = bars;                 // [kStages] x landed + decay factors written
    uint64_t *op_full = st_full + kStages;    // [kStages] transform -> MMA
    uint64_t *st_empty = op_full + kStages;   // [kStages] MMA commit -> producer, prep
    uint64_t *acc_full = st_empty + kStages;  // [4] MMA commit after a run's last block
    uint64_t *acc_empty = acc_full + 4;       // [4] epilogue drained
    uint64_t *b_full = acc_empty + 4;         // [2] B tile landed
    uint64_t *b_empty = b_full + 2;           // [2] MMA commit after the unit's last item
    uint64_t *fin = b_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u0 = lay.first(blockIdx.x), u1 = lay.first(blockIdx.x + 1);
    const int cnt = kPairHeads * (u1 - u0);
    if (cnt <= 0) return;
    const int nk = lay.nk, NQ = H / kPairHeads, hpg = H / G;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&st_full[i], 2);  // the producer's expect_tx arrive + the prep warp
            mbar_init(&op_full[i], kXform);
            mbar_init(&st_empty[i], 1);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kEpi);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
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
    grid_dependency_wait();
    dt = after_wait(dt);
    A_log = after_wait(A_log);
    dt_bias = after_wait(dt_bias);
    decay_out = after_wait(decay_out);
    status = after_wait(status);
    // the first kernel of the call: its status word starts clean, unless the caller keeps one
    // word across several calls (the varlen prefill)
    if (reset_status && blockIdx.x == 0 && tid == 0) *status = SSD_OK;

    auto stage = [&](int j) { return smem + kOffStage + (uint32_t)(j % kStages) * kStageBytes; };
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
            RevItems it(u0, u1, nk);
            int units = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int ch = it.u / nk, k = it.u - ch * nk;
                const int b = ch / NQ, h = (ch - b * NQ) * kPairHeads + it.hh, g = h / hpg;
                if (it.hh == 0) {  // a new unit: its B tile into slot units & 1
                    const int bs = units & 1;
                    if (units >= 2 && !wait(&b_empty[bs], ((units >> 1) - 1) & 1)) break;
                    mbar_arrive_expect_tx(&b_full[bs], 2 * kBox);
                    tma_load_3d(smem + kOffB + bs * 2 * kBox, &tm_b, g * N, k * R, b, &b_full[bs]);
                    tma_load_3d(smem + kOffB + bs * 2 * kBox + kBox, &tm_b, g * N + 64, k * R, b, &b_full[bs]);
                    ++units;
                }
                const int s = j % kStages;
                if (j >= kStages && !wait(&st_empty[s], ((j / kStages) - 1) & 1)) break;
                mbar_arrive_expect_tx(&st_full[s], kBox);
                tma_load_3d(stage(j), &tm_x, h * P, k * R, b, &st_full[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true, true);  // N = [hi | lo]
            RevItems it(u0, u1, nk);
            int units = 0;
            for (int j = 0; j < cnt; ++j, it.next()) {
                const int s = j % kStages;
                const int a = (it.r & 1) * kPairHeads + it.hh;  // accumulator of (run parity, head)
                const int bs = (units - (it.hh == 0 ? 0 : 1)) & 1;
                if (it.hh == 0) {
                    if (!wait(&b_full[units & 1], (units >> 1) & 1)) break;
                    ++units;
                }
                if (!wait(&op_full[s], (j / kStages) & 1)) break;
                if (it.run_first() && it.r >= 2 && !wait(&acc_empty[a], ((it.r >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint64_t da = desc_mnmajor_sw128(smem_u32(smem + kOffB + bs * 2 * kBox), kBox);
                const uint64_t dh = desc_mnmajor_sw128(smem_u32(stage(j)), kBox);  // [hi | lo] at LBO kBox
                const uint32_t d = tmem + (uint32_t)(a * 128);
#pragma unroll
                for (int kk = 0; kk < R / 16; ++kk)
                    mma_ss(d, desc_add(da, kk * 2048), desc_add(dh, kk * 2048), idesc,
                           (kk > 0 || !it.run_first()) ? 1u : 0u);
                mma_commit(&st_empty[s]);
                if (it.hh == kPairHeads - 1) mma_commit(&b_empty[bs]);
                if (it.run_last()) mma_commit(&acc_full[a]);
            }
            mma_commit(fin);
            mbar_wait(fin, 0, status);
        }
    } else if (warp < kXformWarp) {
        // ---------------------------------------------------------------- decay factors
        // warp 2 + hh serves head hh's items (j = hh, hh + 2, ...).  Lane i holds tokens 4i .. 4i+3
        // of the block.  The weight of token s is dt_s * 2^lw_s with
        //   lw_s = log2(dt_s) + (suffix sum of dA after s in the block + dA of the run's later
        //          blocks) * log2(e);
        // the suffix sums come from a reversed warp scan, so a lane past the last real token holds
        // exact zeros and the last real token's own suffix is exactly 0.
        const int hh = warp - 2;
        RevItems it(u0, u1, nk), ahead(u0, u1, nk);
        auto load_raw = [&](const RevItems &c, float (&r)[4]) {
            const int ch = c.u / nk, k = c.u - ch * nk;
            const int b = ch / NQ, h = (ch - b * NQ) * kPairHeads + hh;
            const int t0 = k * R + lane * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                r[i] = t0 + i < L ? __bfloat162float(dt[((size_t)b * L + t0 + i) * H + h]) : 0.f;
        };
        if (hh == 1) {
            it.next();
            ahead.next();
        }
        float r0[4];
        load_raw(ahead, r0);  // the strided dt loads of the next item are issued before this one is formed
        ahead.next();
        ahead.next();
        float carry = 0.f;  // dA of the run's blocks already done (those after the current one)
        for (int j = hh; j < cnt; j += kPairHeads) {
            const int ch = it.u / nk, k = it.u - ch * nk;
            const int b = ch / NQ, h = (ch - b * NQ) * kPairHeads + hh;
            const int t0 = k * R + lane * 4;
            float raw[4] = {r0[0], r0[1], r0[2], r0[3]};
            if (j + kPairHeads < cnt) {
                load_raw(ahead, r0);
                ahead.next();
                ahead.next();
            }
            const float bias = dt_bias ? __ldg(dt_bias + h) : 0.f;
            const float A = -expf(__ldg(A_log + h));
            if (it.run_first()) carry = 0.f;
            const int s = j % kStages;
            const bool ok = j < kStages || wait(&st_empty[s], ((j / kStages) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            float d[4], dA[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d[i] = t0 + i < L ? discretise_dt(raw[i], bias, dt_min, dt_max) : 0.f;
                dA[i] = d[i] * A;
            }
            const float run = ((dA[3] + dA[2]) + dA[1]) + dA[0];
            float incl = run;  // sum of run over lanes >= this one
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float nv = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += nv;
            }
            float sfx = __shfl_down_sync(0xffffffffu, incl, 1);  // lanes > this one
            if (lane == 31) sfx = 0.f;
            const float total = __shfl_sync(0xffffffffu, incl, 0);
            float lw[4];
#pragma unroll
            for (int i = 3; i >= 0; --i) {
                lw[i] = log2f(d[i]) + (sfx + carry) * kLog2e;
                sfx += dA[i];
            }
            reinterpret_cast<float4 *>(stage(j) + 2 * kBox)[lane] = make_float4(lw[0], lw[1], lw[2], lw[3]);
            carry += total;
            if (it.run_last() && lane == 0) decay_out[lay.slot(it.rs, blockIdx.x) * kPairHeads + hh] = carry * kLog2e;
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_full[s]);
            it.next();
            it.next();
        }
    } else if (warp < kEpiWarp) {
        // ---------------------------------------------------------------- transform
        const int tw = warp - kXformWarp;  // rows [16 tw, 16 tw + 16)
        for (int j = 0; j < cnt; ++j) {
            const int s = j % kStages;
            if (!__all_sync(0xffffffffu, wait(&st_full[s], (j / kStages) & 1))) break;
            uint8_t *xt = stage(j);
            uint8_t *lo = xt + kBox;
            const float *lwr = reinterpret_cast<const float *>(xt + 2 * kBox);
            const float wl = lane < 16 ? ex2_approx(lwr[tw * 16 + lane]) : 0.f;
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
        // per run, head 0 then head 1: TMEM lane quarter (warp % 4) = rows n, column half = p range
        const int quarter = warp & 3, half = (warp - kEpiWarp) >> 2;
        const int n = quarter * 32 + lane;
        const bool leader = warp == kEpiWarp && lane == 0;
        uint8_t *box = smem + kOffOut + half * kBox;
        RevItems it(u0, u1, nk);
        for (int j = 0; j < cnt; ++j, it.next()) {
            if (!it.run_last()) continue;  // only a run's last block completes an accumulator
            const int a = (it.r & 1) * kPairHeads + it.hh;
            const bool ok = __all_sync(0xffffffffu, wait(&acc_full[a], (it.r >> 1) & 1));
            float v[32];
            if (ok) {
                tc_fence_after();
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
            if (leader) bulk_wait_read();
            if (!named_barrier_and(kEpiBar, kEpi * 32, ok)) break;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<float4 *>(box + sw128_offset(n, c)) =
                    make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_proxy_async_smem();
            named_barrier(kEpiBar, kEpi * 32);
            if (leader) {
                const int row = (lay.slot(it.rs, blockIdx.x) * kPairHeads + it.hh) * N;
                tma_store_2d(&tm_s, smem + kOffOut, 0, row);
                tma_store_2d(&tm_s, smem + kOffOut + kBox, 32, row);
                bulk_commit();
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

cudaError_t launch_run_state_tc(const void *x, const void *Bm, const void *dt, const float *A_log,
                                const float *dt_bias, float dt_min, float dt_max, float *slots, float *decays,
                                int *status, bool reset_status, int B, int L, int H, int G, int64_t x_row,
                                int64_t bc_row, const RunLayout &lay, cudaStream_t st) {
    using namespace rst;
    CUtensorMap tm_x, tm_b, tm_s;
    cudaError_t e = make_tmap_bf16_3d(&tm_x, x, (uint64_t)H * P, (uint64_t)L, (uint64_t)B, (uint64_t)x_row * 2,
                                      (uint64_t)L * x_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_3d(&tm_b, Bm, (uint64_t)G * N, (uint64_t)L, (uint64_t)B, (uint64_t)bc_row * 2,
                          (uint64_t)L * bc_row * 2, 64, R, 1);
    if (e != cudaSuccess) return e;
    // every slot's two heads' S^T as rows of 64 fp32: boxes of 32 columns x 128 rows
    e = make_tmap_f32_2d(&tm_s, slots, (uint64_t)P, (uint64_t)lay.slots() * kPairHeads * N, (uint64_t)P * 4, 32, R);
    if (e != cudaSuccess) return e;
    e = raise_smem_limit<run_state_tc_kernel>((int)kSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(run_state_tc_kernel, dim3(lay.grid), dim3(kThreads), kSmem, st, tm_x, tm_b, tm_s,
                      (const __nv_bfloat16 *)dt, A_log, dt_bias, dt_min, dt_max, decays, status, reset_status ? 1 : 0, L, H, G,
                      lay);
}

}  // namespace ssd
