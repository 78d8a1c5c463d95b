// api.cu -- the extern "C" boundary of libmamba_ssd.so: argument validation, workspace
// carving and kernel sequencing.  Every check happens before anything is enqueued.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "launch.h"

namespace {

thread_local int g_last_cuda_error = 0;

// ---- profiling hooks: launch counter and optional per-kernel CUDA-event timing ----
const char *const kKernelNames[] = {"decay_prep",  "chunk_state",   "state_pass",  "chunk_scan",
                                    "decode_step", "causal_conv1d", "decode_conv", "gated_rmsnorm",
                                    "run_state",   "run_pass",      "chunk_scan_fused", "segment_decay",
                                    "state_combine"};
enum KernelId {
    K_DECAY = 0,
    K_STATE,
    K_PASS,
    K_SCAN,
    K_DECODE,
    K_CONV,
    K_DCONV,
    K_NORM,
    K_RSTATE,
    K_RPASS,
    K_FSCAN,
    K_SEGDECAY,
    K_COMBINE,
    K_COUNT
};

std::atomic<long long> g_launches{0};
std::atomic<int> g_timer_on{0};
std::mutex g_timer_mu;
std::vector<cudaEvent_t> g_event_pool;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_timed[K_COUNT];

cudaEvent_t pooled_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Runs one launcher, counting it and (when the timer is on) bracketing it with events.
template <typename F>
cudaError_t timed_launch(KernelId id, cudaStream_t st, F &&launch) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_timer_on.load(std::memory_order_relaxed)) return launch();
    cudaEvent_t a, b;
    {
        std::lock_guard<std::mutex> lk(g_timer_mu);
        a = pooled_event();
        b = pooled_event();
    }
    if (!a || !b) {  // give back whichever event was made
        std::lock_guard<std::mutex> lk(g_timer_mu);
        if (a) g_event_pool.push_back(a);
        if (b) g_event_pool.push_back(b);
        return cudaErrorMemoryAllocation;
    }
    cudaEventRecord(a, st);
    const cudaError_t e = launch();
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_timer_mu);
    g_timed[id].emplace_back(a, b);
    return e;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool opt_aligned16(const void *p) { return p == nullptr || aligned16(p); }

inline int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    g_last_cuda_error = (int)e;
    return SSD_ERR_CUDA;
}

}  // namespace

namespace ssd {
bool pdl_enabled() {
    static const bool on = [] {
        const char *v = getenv("SSD_PDL");
        return !(v && v[0] == '0');
    }();
    return on;
}
}  // namespace ssd

namespace {
// Tensor-core kernels are used wherever they apply, unless SSD_PREFILL_KERNELS=simt is set in
// the environment (then every shape runs on the float32 CUDA-core kernels).  By default the
// tensor-core path is the block-state one (per-block states through memory, one state pass);
// SSD_PREFILL_KERNELS=fused selects the run-carrying kernels for the shapes they support
// (each head pair's state carried through runs of blocks on chip: a fraction of the memory
// traffic, but slower on B200 as measured, so not the default).
bool use_tensor_cores() {
    static const bool on = [] {
        const char *v = getenv("SSD_PREFILL_KERNELS");
        return !(v && strcmp(v, "simt") == 0);
    }();
    return on;
}
bool use_fused() {
    static const bool on = [] {
        const char *v = getenv("SSD_PREFILL_KERNELS");
        return v && strcmp(v, "fused") == 0;
    }();
    return on;
}
bool fused_path(int dtype, int L, int P, int N, int H, int G) {
    return L > 0 && use_fused() && ssd::prefill_fused_supported(dtype, P, N, H, G);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

inline bool is_pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

int check_dt_range(float dt_min, float dt_max) {
    if (isnan(dt_min) || isnan(dt_max) || dt_min < 0.f || dt_min > dt_max) return SSD_ERR_INVALID_ARG;
    return SSD_OK;
}

// Shape checks shared by the prefill size query and the call itself.
int check_prefill_shape(int B, int L, int H, int P, int G, int N, int chunk, int dtype) {
    if (B < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || chunk <= 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (H % G != 0) return SSD_ERR_INVALID_ARG;
    if (P != 64) return SSD_ERR_UNSUPPORTED;
    if (N != 16 && N != 32 && N != 64 && N != 128) return SSD_ERR_UNSUPPORTED;
    if (chunk != 64 && chunk != 128 && chunk != 256 && chunk != 512) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

}  // namespace

namespace ssd {

constexpr size_t kStatusSlot = 256;

size_t prefill_workspace_bytes(int B, int L, int H, int P, int N, int block, bool transposed_bf16) {
    const size_t nb = (size_t)cdiv(L, block), Lp = nb * block;
    const size_t per_tok = align_up(sizeof(float) * (size_t)B * H * Lp, 256);
    const size_t states = align_up(sizeof(float) * (size_t)B * nb * H * P * N, 256);
    const size_t hT = transposed_bf16 ? align_up(2 * (size_t)B * nb * H * P * N, 256) : 0;
    return kStatusSlot + 2 * per_tok + states + hT;
}

PrefillWorkspace carve_prefill_workspace(void *base, int B, int L, int H, int P, int N, int block,
                                         bool transposed_bf16) {
    const size_t nb = (size_t)cdiv(L, block), Lp = nb * block;
    const size_t per_tok = align_up(sizeof(float) * (size_t)B * H * Lp, 256);
    const size_t states = align_up(sizeof(float) * (size_t)B * nb * H * P * N, 256);
    char *p = static_cast<char *>(base);
    PrefillWorkspace w;
    w.status = reinterpret_cast<int *>(p);
    p += kStatusSlot;
    w.dtf = reinterpret_cast<float *>(p);
    w.acs = reinterpret_cast<float *>(p + per_tok);
    w.states = reinterpret_cast<float *>(p + 2 * per_tok);
    w.hT = transposed_bf16 ? reinterpret_cast<__nv_bfloat16 *>(p + 2 * per_tok + states) : nullptr;
    return w;
}

RunLayout fused_layout(int B, int L, int H, int num_sms) {
    RunLayout lay;
    lay.nk = cdiv(L, kTcBlock);
    lay.nch = B * (H / kPairHeads);
    lay.U = lay.nch * lay.nk;
    int g = num_sms < kMaxCtas ? num_sms : kMaxCtas;
    lay.grid = lay.U < g ? lay.U : g;
    return lay;
}

// sized for the largest grid the kernels may use (kMaxCtas), whatever the device
size_t fused_workspace_bytes(int B, int L, int H) {
    const RunLayout lay = fused_layout(B, L, H, kMaxCtas);
    const size_t slots = (size_t)lay.slots() * kPairHeads;
    return kStatusSlot + align_up(slots * 128 * 64 * sizeof(float), 256) + align_up(slots * sizeof(float), 256);
}

FusedWorkspace carve_fused_workspace(void *base, int B, int L, int H) {
    const RunLayout lay = fused_layout(B, L, H, kMaxCtas);
    const size_t slots = (size_t)lay.slots() * kPairHeads;
    char *p = static_cast<char *>(base);
    FusedWorkspace w;
    w.status = reinterpret_cast<int *>(p);
    w.slots = reinterpret_cast<float *>(p + kStatusSlot);
    w.decays = reinterpret_cast<float *>(p + kStatusSlot + align_up(slots * 128 * 64 * sizeof(float), 256));
    return w;
}

}  // namespace ssd

namespace {
// Bytes a prefill needs on the path its shape runs (the environment switches, read once per
// process, decide the path the same way for the query and the call).
size_t prefill_query_bytes(int B, int L, int H, int P, int G, int N, int chunk, int dtype) {
    if (fused_path(dtype, L, P, N, H, G)) return ssd::fused_workspace_bytes(B, L, H);
    size_t need = ssd::prefill_workspace_bytes(B, L, H, P, N, chunk, false);
    if (use_tensor_cores() && ssd::prefill_tc_supported(dtype, P, N)) {
        const size_t tc = ssd::prefill_workspace_bytes(B, L, H, P, N, ssd::kTcBlock, true);
        if (tc > need) need = tc;
    }
    return need;
}

// A packed varlen batch: its non-empty sequences (m), their 128-token blocks in all, its
// longest sequence.  Checks that the cumulative lengths start at 0 and never decrease.
struct VarlenPlan {
    int m = 0, nblocks = 0, max_len = 0;
};
int varlen_plan(const int *cu, int n_seq, VarlenPlan &p) {
    if (cu[0] != 0) return SSD_ERR_INVALID_ARG;
    p = VarlenPlan();
    for (int i = 0; i < n_seq; ++i) {
        if (cu[i + 1] < cu[i]) return SSD_ERR_INVALID_ARG;
        const int len = cu[i + 1] - cu[i];
        if (len > p.max_len) p.max_len = len;
        if (len > 0) {
            ++p.m;
            p.nblocks += ssd::cdiv(len, ssd::kTcBlock);
        }
    }
    return SSD_OK;
}
// The tensor-core path runs a packed batch in one pass; the CUDA-core and the run-carrying
// kernels take its sequences one at a time.
bool varlen_one_pass(int dtype, int P, int N) {
    return use_tensor_cores() && !use_fused() && ssd::prefill_tc_supported(dtype, P, N);
}
// One pass: the block-major prefill workspace of all the batch's blocks, then the table
// (tok0, blk0, seq: m + 1 ints each, each in its own 256-byte-aligned slot).
size_t varlen_table_offset(const VarlenPlan &p, int H, int P, int N) {
    return ssd::prefill_workspace_bytes(1, p.nblocks * ssd::kTcBlock, H, P, N, ssd::kTcBlock, true);
}
size_t varlen_query_bytes(const VarlenPlan &p, int H, int P, int G, int N, int chunk, int dtype) {
    if (!varlen_one_pass(dtype, P, N)) return prefill_query_bytes(1, p.max_len, H, P, G, N, chunk, dtype);
    return varlen_table_offset(p, H, P, N) + 3 * ssd::align_up(sizeof(int) * (size_t)(p.m + 1), 256);
}

}  // namespace

extern "C" {

const char *ssd_status_string(int status) {
    switch (status) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size)";
        case SSD_ERR_UNSUPPORTED: return "shape or dtype not supported by the kernels";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
        case SSD_ERR_CUDA: return "CUDA error (see ssd_last_cuda_error)";
        case SSD_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        default: return "unknown status";
    }
}

int ssd_last_cuda_error(void) { return g_last_cuda_error; }

int ssd_abi_version(void) { return 5; }

size_t ssd_chunk_scan_workspace_size(int B, int L, int H, int P, int G, int N, int chunk,
                                     int dtype) {
    if (check_prefill_shape(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    if (B == 0) return 0;
    return prefill_query_bytes(B, L, H, P, G, N, chunk, dtype);
}

}  // extern "C"

namespace {
// The prefill.  reset_status: the call's first kernel resets the workspace status word (a
// single call); the varlen prefill resets it once itself and keeps it across its sequences.
// x_row, bc_row: elements between consecutive tokens of x and of B / C (H*P and G*N when
// dense; Cc when x, B and C are views into one conv output [.., Cc]).  y == NULL computes the
// state only (h_final), skipping the output kernels.
// The tensor-core prefill's three launches over an equal-length batch (vl.n = 0: B sequences
// of L tokens) or a packed varlen batch (B = 1, L = the packed token count, vl its table), with
// nblocks 128-token blocks in all.
int tc_prefill(const void *x, const void *dt, const float *A_log, const void *Bm, const void *Cm, const float *D,
               const float *dt_bias, float dt_min, float dt_max, const float *h0, void *y, float *h_final, int B,
               int L, int H, int P, int G, int N, const ssd::PrefillWorkspace &ws, const ssd::Varlen &vl, int nblocks,
               bool reset_status, int64_t x_row, int64_t bc_row, cudaStream_t st) {
    const int blk = ssd::kTcBlock;
    cudaError_t e = cudaSuccess;
    if (nblocks > 0) {
        // the state kernel also forms the decay factors (step a1) of the items it owns
        e = timed_launch(K_STATE, st, [&] {
            return ssd::launch_chunk_state_tc(x, Bm, dt, A_log, dt_bias, dt_min, dt_max, ws.dtf, ws.acs, ws.states,
                                              ws.status, reset_status, B, L, H, G, x_row, bc_row, vl, nblocks,
                                              sm_count(), st);
        });
        if (e != cudaSuccess) return cuda_status(e);
    }
    e = timed_launch(K_PASS, st, [&] {
        return ssd::launch_state_pass_t(ws.states, ws.acs, h0, h_final, ws.hT, B, L, H, P, N, blk, vl, nblocks, st);
    });
    if (e != cudaSuccess) return cuda_status(e);
    if (nblocks > 0 && y) {
        e = timed_launch(K_SCAN, st, [&] {
            return ssd::launch_chunk_scan_tc(x, Bm, Cm, ws.dtf, ws.acs, ws.hT, D, y, ws.status, B, L, H, G, x_row,
                                             bc_row, vl, nblocks, sm_count(), st);
        });
        if (e != cudaSuccess) return cuda_status(e);
    }
    return SSD_OK;
}

int prefill(const void *x, const void *dt, const float *A_log, const void *Bm, const void *Cm, const float *D,
            const float *dt_bias, float dt_min, float dt_max, const float *h0, void *y, float *h_final, int B, int L,
            int H, int P, int G, int N, int chunk, int dtype, void *workspace, size_t workspace_bytes, void *stream,
            bool reset_status, int64_t x_row, int64_t bc_row) {
    int s = check_prefill_shape(B, L, H, P, G, N, chunk, dtype);
    if (s != SSD_OK) return s;
    if ((s = check_dt_range(dt_min, dt_max)) != SSD_OK) return s;
    if (B == 0) return SSD_OK;
    if (!A_log || !aligned16(A_log) || !opt_aligned16(D) || !opt_aligned16(dt_bias) ||
        !opt_aligned16(h0) || !opt_aligned16(h_final))
        return SSD_ERR_INVALID_ARG;
    if (L > 0) {
        if (!x || !dt || !Bm || (y && !Cm)) return SSD_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(dt) || !aligned16(Bm) || !opt_aligned16(Cm) || !opt_aligned16(y))
            return SSD_ERR_INVALID_ARG;
    }
    const bool want_y = y != nullptr;
    const size_t need = prefill_query_bytes(B, L, H, P, G, N, chunk, dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (fused_path(dtype, L, P, N, H, G)) {
        // fused tensor-core path: run states, the pass over runs, the scan carrying the states
        const ssd::RunLayout lay = ssd::fused_layout(B, L, H, sm_count());
        ssd::FusedWorkspace ws = ssd::carve_fused_workspace(workspace, B, L, H);
        e = timed_launch(K_RSTATE, st, [&] {
            return ssd::launch_run_state_tc(x, Bm, dt, A_log, dt_bias, dt_min, dt_max, ws.slots, ws.decays,
                                            ws.status, reset_status, B, L, H, G, x_row, bc_row, lay, st);
        });
        if (e != cudaSuccess) return cuda_status(e);
        e = timed_launch(K_RPASS, st,
                         [&] { return ssd::launch_run_pass(ws.slots, ws.decays, h0, h_final, B, H, lay, st); });
        if (e != cudaSuccess || !want_y) return cuda_status(e);
        e = timed_launch(K_FSCAN, st, [&] {
            return ssd::launch_chunk_scan_fused(x, Bm, Cm, dt, A_log, dt_bias, dt_min, dt_max, D, ws.slots, y,
                                                ws.status, B, L, H, G, x_row, bc_row, lay, st);
        });
        return cuda_status(e);
    }
    if (use_tensor_cores() && ssd::prefill_tc_supported(dtype, P, N)) {
        // tensor-core path: 128-token blocks, block states in fp32, h_prev^T in bf16
        const int blk = ssd::kTcBlock;
        ssd::PrefillWorkspace ws = ssd::carve_prefill_workspace(workspace, B, L, H, P, N, blk, true);
        return tc_prefill(x, dt, A_log, Bm, Cm, D, dt_bias, dt_min, dt_max, h0, y, h_final, B, L, H, P, G, N,
                          ws, ssd::Varlen{nullptr, nullptr, nullptr, 0}, B * ssd::cdiv(L, blk), reset_status, x_row,
                          bc_row, st);
    }
    // CUDA-core path: the caller's chunk, fp32 throughout
    ssd::PrefillWorkspace ws = ssd::carve_prefill_workspace(workspace, B, L, H, P, N, chunk, false);
    if (L > 0) {
        e = timed_launch(K_DECAY, st, [&] {
            return ssd::launch_decay_prep(dtype, dt, A_log, dt_bias, dt_min, dt_max, ws.dtf, ws.acs,
                                          reset_status ? ws.status : nullptr, B, L, H, chunk, st);
        });
        if (e != cudaSuccess) return cuda_status(e);
        e = timed_launch(K_STATE, st, [&] {
            return ssd::launch_chunk_state(dtype, x, Bm, ws.dtf, ws.acs, ws.states, B, L, H, G, N, chunk, x_row,
                                           bc_row, st);
        });
        if (e != cudaSuccess) return cuda_status(e);
    }
    e = timed_launch(K_PASS, st, [&] {
        return ssd::launch_state_pass(ws.states, ws.acs, h0, h_final, B, L, H, P, N, chunk, st);
    });
    if (e != cudaSuccess) return cuda_status(e);
    if (L > 0 && want_y) {
        e = timed_launch(K_SCAN, st, [&] {
            return ssd::launch_chunk_scan(dtype, x, Bm, Cm, ws.dtf, ws.acs, ws.states, D, y, B, L, H, G, N,
                                          chunk, x_row, bc_row, st);
        });
        if (e != cudaSuccess) return cuda_status(e);
    }
    return SSD_OK;
}

}  // namespace

extern "C" {

int ssd_chunk_scan_fwd(const void *x, const void *dt, const float *A_log, const void *Bm, const void *Cm,
                       const float *D, const float *dt_bias, float dt_min, float dt_max, const float *h0, void *y,
                       float *h_final, int B, int L, int H, int P, int G, int N, int chunk, int dtype,
                       void *workspace, size_t workspace_bytes, void *stream) {
    return prefill(x, dt, A_log, Bm, Cm, D, dt_bias, dt_min, dt_max, h0, y, h_final, B, L, H, P, G, N, chunk,
                   dtype, workspace, workspace_bytes, stream, true, (int64_t)H * P, (int64_t)G * N);
}

// The prefill workspace first (so its status word is the workspace's first word), then the
// conv output u [B, L, Cc].
namespace {
size_t conv_out_bytes(int B, int L, int Cc, int dtype) {
    return ssd::align_up((size_t)B * L * Cc * (dtype == SSD_DTYPE_BF16 ? 2 : 4), 256);
}
int check_conv_shape(int B, int L, int Cc, int K) {
    if (K < 2 || K > 8 || Cc % 8 != 0) return SSD_ERR_UNSUPPORTED;
    if (B > 65535 || L > 65535 * 32) return SSD_ERR_UNSUPPORTED;  // grid z; 32-token strips on grid y
    return SSD_OK;
}
}  // namespace

size_t ssd_conv_chunk_scan_workspace_size(int B, int L, int H, int P, int G, int N, int K, int chunk, int dtype) {
    if (check_prefill_shape(B, L, H, P, G, N, chunk, dtype) != SSD_OK || K <= 0) return 0;
    const int Cc = H * P + 2 * G * N;
    if (check_conv_shape(B, L, Cc, K) != SSD_OK || B == 0) return 0;
    return prefill_query_bytes(B, L, H, P, G, N, chunk, dtype) + conv_out_bytes(B, L, Cc, dtype);
}

int ssd_conv_chunk_scan_fwd(const void *xBC, const void *conv_w, const void *conv_b, const void *dt,
                            const float *A_log, const float *D, const float *dt_bias, float dt_min, float dt_max,
                            const float *h0, void *y, float *h_final, void *conv_state_out, int B, int L, int H,
                            int P, int G, int N, int K, int chunk, int dtype, void *workspace, size_t workspace_bytes,
                            void *stream) {
    int s = check_prefill_shape(B, L, H, P, G, N, chunk, dtype);
    if (s != SSD_OK) return s;
    if (K <= 0) return SSD_ERR_INVALID_ARG;
    const int Cc = H * P + 2 * G * N;
    if ((s = check_conv_shape(B, L, Cc, K)) != SSD_OK) return s;
    if ((s = check_dt_range(dt_min, dt_max)) != SSD_OK) return s;
    if (B == 0) return SSD_OK;
    if (!conv_w || !aligned16(conv_w) || !opt_aligned16(conv_b) || !opt_aligned16(conv_state_out) || !A_log ||
        !aligned16(A_log) || !opt_aligned16(D) || !opt_aligned16(dt_bias) || !opt_aligned16(h0) ||
        !opt_aligned16(h_final))
        return SSD_ERR_INVALID_ARG;
    if (L > 0 && (!xBC || !dt || !y || !aligned16(xBC) || !aligned16(dt) || !aligned16(y))) return SSD_ERR_INVALID_ARG;
    const size_t pre_bytes = prefill_query_bytes(B, L, H, P, G, N, chunk, dtype);
    const size_t need = pre_bytes + conv_out_bytes(B, L, Cc, dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t e = dtype == SSD_DTYPE_BF16 ? 2 : 4;
    char *u = static_cast<char *>(workspace) + pre_bytes;
    cudaError_t ce = cudaSuccess;
    if (L > 0) {
        ce = timed_launch(K_CONV, st, [&] {
            return ssd::launch_causal_conv1d(dtype, xBC, conv_w, conv_b, u, conv_state_out, B, L, Cc, K, st);
        });
    } else if (conv_state_out) {  // empty prefix: the cache is all zeros
        ce = cudaMemsetAsync(conv_state_out, 0, (size_t)B * Cc * (K - 1) * e, st);
    }
    if (ce != cudaSuccess) return cuda_status(ce);
    // x, B and C are strided views of u (token rows Cc elements apart): no split, no copy
    return prefill(u, dt, A_log, u + (size_t)H * P * e, u + ((size_t)H * P + (size_t)G * N) * e, D, dt_bias, dt_min,
                   dt_max, h0, y, h_final, B, L, H, P, G, N, chunk, dtype, workspace, pre_bytes, stream, true, Cc, Cc);
}

int ssd_segment_decay(const void *dt, const float *A_log, const float *dt_bias, float dt_min, float dt_max,
                      float *log2_decay, int B, int L, int H, int dtype, void *stream) {
    if (B < 0 || L < 0 || H <= 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    int s = check_dt_range(dt_min, dt_max);
    if (s != SSD_OK) return s;
    if (B == 0) return SSD_OK;
    if (!A_log || !log2_decay || !aligned16(A_log) || !aligned16(log2_decay) || !opt_aligned16(dt_bias))
        return SSD_ERR_INVALID_ARG;
    if (L > 0 && (!dt || !aligned16(dt))) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(timed_launch(K_SEGDECAY, st, [&] {
        return ssd::launch_segment_decay(dtype, dt, A_log, dt_bias, dt_min, dt_max, log2_decay, B, L, H, st);
    }));
}

int ssd_state_combine(const float *states, const float *log2_decays, const float *h0, float *out, int r, int B, int H,
                      int P, int N, void *stream) {
    if (r < 0 || B < 0 || H <= 0 || P <= 0 || N <= 0) return SSD_ERR_INVALID_ARG;
    if (((size_t)P * N) % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (B == 0) return SSD_OK;
    if (!out || !aligned16(out) || !opt_aligned16(h0)) return SSD_ERR_INVALID_ARG;
    if (r > 0 && (!states || !log2_decays || !aligned16(states) || !aligned16(log2_decays))) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(timed_launch(K_COMBINE, st, [&] {
        return ssd::launch_state_combine(states, log2_decays, h0, out, r, B, H, P, N, st);
    }));
}

int ssd_chunk_scan_varlen_fwd(const void *x, const void *dt, const float *A_log, const void *Bm,
                              const void *Cm, const float *D, const float *dt_bias, float dt_min,
                              float dt_max, const float *h0, void *y, float *h_final,
                              const int *cu_seqlens, int n_seq, int H, int P, int G, int N, int chunk,
                              int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (n_seq < 0 || (n_seq > 0 && !cu_seqlens)) return SSD_ERR_INVALID_ARG;
    if (n_seq == 0) return SSD_OK;
    VarlenPlan plan;
    int s = varlen_plan(cu_seqlens, n_seq, plan);
    if (s != SSD_OK) return s;
    s = check_prefill_shape(1, plan.max_len, H, P, G, N, chunk, dtype);
    if (s != SSD_OK) return s;
    if ((s = check_dt_range(dt_min, dt_max)) != SSD_OK) return s;
    const size_t e = dtype == SSD_DTYPE_BF16 ? 2 : 4;
    const bool any_tokens = cu_seqlens[n_seq] > 0;
    if (!A_log || !aligned16(A_log) || !opt_aligned16(D) || !opt_aligned16(dt_bias) || !opt_aligned16(h0) ||
        !opt_aligned16(h_final))
        return SSD_ERR_INVALID_ARG;
    if (any_tokens && (!x || !dt || !Bm || !Cm || !y || !aligned16(x) || !aligned16(dt) || !aligned16(Bm) ||
                       !aligned16(Cm) || !aligned16(y)))
        return SSD_ERR_INVALID_ARG;
    const bool one_pass = varlen_one_pass(dtype, P, N);
    // the per-sequence path hands each sequence's rows to the prefill as its own arrays, which
    // must start on a 16-byte boundary (x, y, B, C always do for the supported P and N; dt does
    // when H * e is a multiple of 16 or the offsets happen to be)
    if (!one_pass)
        for (int i = 0; i < n_seq; ++i)
            if (((size_t)cu_seqlens[i] * H * e) % 16 != 0 || ((size_t)cu_seqlens[i] * G * N * e) % 16 != 0)
                return SSD_ERR_UNSUPPORTED;
    const size_t need = varlen_query_bytes(plan, H, P, G, N, chunk, dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t state = (size_t)H * P * N;
    if (one_pass) {
        // every argument is valid.  The empty sequences hand h0 (or zeros) straight through;
        // the others run as one packed batch: the table of its non-empty sequences into the
        // workspace, then the three tensor-core launches over all of their blocks.
        cudaError_t ce = cudaSuccess;
        for (int i = 0; i < n_seq && h_final; ++i) {
            if (cu_seqlens[i + 1] != cu_seqlens[i]) continue;
            ce = h0 ? cudaMemcpyAsync(h_final + i * state, h0 + i * state, state * sizeof(float),
                                      cudaMemcpyDeviceToDevice, st)
                    : cudaMemsetAsync(h_final + i * state, 0, state * sizeof(float), st);
            if (ce != cudaSuccess) return cuda_status(ce);
        }
        ssd::PrefillWorkspace ws =
            ssd::carve_prefill_workspace(workspace, 1, plan.nblocks * ssd::kTcBlock, H, P, N, ssd::kTcBlock, true);
        if (plan.m == 0) {  // nothing to scan: the call's status word is still this call's
            return cuda_status(cudaMemsetAsync(ws.status, 0, sizeof(int), st));
        }
        int *tab = reinterpret_cast<int *>(static_cast<char *>(workspace) + varlen_table_offset(plan, H, P, N));
        const size_t slot = ssd::align_up(sizeof(int) * (size_t)(plan.m + 1), 256) / sizeof(int);
        int *tok0 = tab, *blk0 = tab + slot, *seq = tab + 2 * slot;
        ssd::VarlenTableChunk c;
        c.base = c.count = 0;
        int blocks = 0;
        auto flush = [&]() -> cudaError_t {
            cudaError_t r = c.count ? ssd::launch_varlen_table(c, tok0, blk0, seq, st) : cudaSuccess;
            c.base += c.count;
            c.count = 0;
            return r;
        };
        for (int i = 0; i <= n_seq; ++i) {  // entries j = 0 .. m (the last one the end sentinel)
            const bool end = i == n_seq;
            if (!end && cu_seqlens[i + 1] == cu_seqlens[i]) continue;
            c.tok0[c.count] = cu_seqlens[i];
            c.blk0[c.count] = blocks;
            c.seq[c.count] = end ? 0 : i;
            ++c.count;
            if (!end) blocks += ssd::cdiv(cu_seqlens[i + 1] - cu_seqlens[i], ssd::kTcBlock);
            if (c.count == ssd::kVarlenChunk + 1 && (ce = flush()) != cudaSuccess) return cuda_status(ce);
        }
        if ((ce = flush()) != cudaSuccess) return cuda_status(ce);
        const ssd::Varlen vl{tok0, blk0, seq, plan.m};
        return tc_prefill(x, dt, A_log, Bm, Cm, D, dt_bias, dt_min, dt_max, h0, y, h_final, 1, cu_seqlens[n_seq], H,
                          P, G, N, ws, vl, plan.nblocks, true, (int64_t)H * P, (int64_t)G * N, st);
    }
    // every argument is valid: run each sequence through the prefill, in order on the stream,
    // sharing the workspace (each call's kernels start after the previous call's have ended).
    // The status word is reset once here and kept across the sequences, so that a timeout in
    // any of them is what ssd_chunk_scan_status reports for the call.
    cudaError_t e0 = cudaMemsetAsync(workspace, 0, sizeof(int), st);
    if (e0 != cudaSuccess) return cuda_status(e0);
    for (int i = 0; i < n_seq; ++i) {
        const size_t t0 = (size_t)cu_seqlens[i];
        const int len = cu_seqlens[i + 1] - cu_seqlens[i];
        const char *xb = static_cast<const char *>(x), *dtb = static_cast<const char *>(dt);
        const char *bb = static_cast<const char *>(Bm), *cb = static_cast<const char *>(Cm);
        char *yb = static_cast<char *>(y);
        s = prefill(xb ? xb + t0 * H * P * e : nullptr, dtb ? dtb + t0 * H * e : nullptr, A_log,
                    bb ? bb + t0 * G * N * e : nullptr, cb ? cb + t0 * G * N * e : nullptr, D, dt_bias, dt_min, dt_max,
                    h0 ? h0 + i * state : nullptr, yb ? yb + t0 * H * P * e : nullptr,
                    h_final ? h_final + i * state : nullptr, 1, len, H, P, G, N, chunk, dtype, workspace,
                    workspace_bytes, stream, false, (int64_t)H * P, (int64_t)G * N);
        if (s != SSD_OK) return s;
    }
    return SSD_OK;
}

size_t ssd_chunk_scan_varlen_workspace_size(const int *cu_seqlens, int n_seq, int H, int P, int G, int N, int chunk,
                                            int dtype) {
    if (n_seq <= 0 || !cu_seqlens) return 0;
    VarlenPlan plan;
    if (varlen_plan(cu_seqlens, n_seq, plan) != SSD_OK) return 0;
    if (check_prefill_shape(1, plan.max_len, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    return varlen_query_bytes(plan, H, P, G, N, chunk, dtype);
}

int ssd_chunk_scan_status(const void *workspace, void *stream) {
    if (!workspace) {  // the built-in scratch of the allocation-free entry, on the current device
        void *p = nullptr;
        const cudaError_t e = ssd::noalloc_scratch(&p);
        if (e != cudaSuccess) return cuda_status(e);
        workspace = p;
    }
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
    int v = 0;
    e = cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    return v;
}

// Decode workspace: a status word (256-byte slot), then u [B][Cc] fp32 (the conv outputs of
// the step), then (dt, a) [B][H] as float2; each part starts on a 256-byte boundary.
namespace {
size_t decode_u_bytes(int B, int H, int P, int G, int N) {
    return ssd::align_up(sizeof(float) * (size_t)B * ((size_t)H * P + 2 * (size_t)G * N), 256);
}
}  // namespace

size_t ssd_decode_workspace_size(int B, int H, int P, int G, int N) {
    if (B <= 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0) return 0;
    return 256 + decode_u_bytes(B, H, P, G, N) + ssd::align_up(2 * sizeof(float) * (size_t)B * H, 256);
}

int ssd_decode_status(const void *workspace, void *stream) {
    if (!workspace) return SSD_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
    int v = 0;
    e = cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    return v;
}

int ssd_decode_step(float *ssm_state, void *conv_state, const void *xBC_t, const void *dt_t,
                    const float *A_log, const float *D, const float *dt_bias, float dt_min,
                    float dt_max, const void *conv_w, const void *conv_b, void *y_t, int B,
                    int H, int P, int G, int N, int K, int dtype, void *workspace,
                    size_t workspace_bytes, void *stream) {
    if (B < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || K <= 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (H % G != 0) return SSD_ERR_INVALID_ARG;
    int s = check_dt_range(dt_min, dt_max);
    if (s != SSD_OK) return s;
    if (P % 16 != 0) return SSD_ERR_UNSUPPORTED;
    if (!is_pow2_in(N, 16, 256)) return SSD_ERR_UNSUPPORTED;
    if (K < 2 || K > 8) return SSD_ERR_UNSUPPORTED;
    if (B > 65535) return SSD_ERR_UNSUPPORTED;  // the batch is the grid's y dimension
    if (B == 0) return SSD_OK;
    if (!ssm_state || !conv_state || !xBC_t || !dt_t || !A_log || !conv_w || !y_t)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(ssm_state) || !aligned16(conv_state) || !aligned16(xBC_t) || !aligned16(dt_t) ||
        !aligned16(A_log) || !aligned16(conv_w) || !aligned16(y_t) || !opt_aligned16(D) ||
        !opt_aligned16(dt_bias) || !opt_aligned16(conv_b))
        return SSD_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < ssd_decode_workspace_size(B, H, P, G, N) || !aligned16(workspace))
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    float *u_ws = reinterpret_cast<float *>(ws + 256);
    float2 *da_ws = reinterpret_cast<float2 *>(ws + 256 + decode_u_bytes(B, H, P, G, N));
    cudaError_t e = timed_launch(K_DCONV, st, [&] {
        return ssd::launch_decode_conv(dtype, conv_state, xBC_t, dt_t, A_log, dt_bias, dt_min, dt_max,
                                       conv_w, conv_b, u_ws, da_ws, B, H, P, G, N, K, st);
    });
    if (e != cudaSuccess) return cuda_status(e);
    e = timed_launch(K_DECODE, st, [&] {
        return ssd::launch_decode_state(dtype, ssm_state, u_ws, da_ws, D, y_t, B, H, P, G, N,
                                        static_cast<int *>(workspace), st);
    });
    return cuda_status(e);
}

int ssd_causal_conv1d_fwd(const void *xBC, const void *conv_w, const void *conv_b, void *out,
                          void *conv_state_out, int B, int L, int Cc, int K, int dtype,
                          void *stream) {
    if (B < 0 || L < 0 || Cc <= 0 || K <= 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (K < 2 || K > 8 || Cc % 8 != 0) return SSD_ERR_UNSUPPORTED;
    if (B > 65535 || L > 65535 * 32) return SSD_ERR_UNSUPPORTED;  // grid z; 32-token strips on grid y
    if (B == 0) return SSD_OK;
    if (!conv_w || !aligned16(conv_w) || !opt_aligned16(conv_b) || !opt_aligned16(conv_state_out))
        return SSD_ERR_INVALID_ARG;
    if (L > 0 && (!xBC || !out || !aligned16(xBC) || !aligned16(out))) return SSD_ERR_INVALID_ARG;
    if (L == 0 && !conv_state_out) return SSD_OK;
    if (L == 0) {
        // empty prefix: the cache is all zeros
        const size_t bytes = (size_t)B * Cc * (K - 1) * (dtype == SSD_DTYPE_BF16 ? 2 : 4);
        return cuda_status(cudaMemsetAsync(conv_state_out, 0, bytes, static_cast<cudaStream_t>(stream)));
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(timed_launch(K_CONV, st, [&] {
        return ssd::launch_causal_conv1d(dtype, xBC, conv_w, conv_b, out, conv_state_out, B, L, Cc, K,
                                         st);
    }));
}

int ssd_gated_rmsnorm_fwd(const void *y, const void *z, const float *w, void *out, int T, int C,
                          int n_groups, float eps, int dtype, void *stream) {
    if (T < 0 || C <= 0 || n_groups <= 0 || C % n_groups != 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_DTYPE_F32 && dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(eps < INFINITY)) return SSD_ERR_INVALID_ARG;  // also rejects NaN
    const int GS = C / n_groups;
    if (GS % 8 != 0 || GS > 32768 || n_groups > 65535) return SSD_ERR_UNSUPPORTED;
    if (T == 0) return SSD_OK;
    if (!y || !z || !w || !out || !aligned16(y) || !aligned16(z) || !aligned16(w) || !aligned16(out))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(timed_launch(K_NORM, st, [&] {
        return ssd::launch_gated_rmsnorm(dtype, y, z, w, out, T, C, n_groups, eps, st);
    }));
}

int ssd_selftest_wait_timeout(int *status, int limit_us, void *stream) {
    if (!status || (reinterpret_cast<uintptr_t>(status) & 3u) || limit_us < 1 || limit_us > 1000000)
        return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_selftest_wait(status, limit_us, static_cast<cudaStream_t>(stream)));
}

long long ssd_kernel_launch_count(void) { return g_launches.load(); }

int ssd_kernel_timer_enable(int on) {
    g_timer_on.store(on ? 1 : 0);
    return SSD_OK;
}

int ssd_kernel_timer_read(const char *name, double *total_ms, long long *launches) {
    if (!name) return SSD_ERR_INVALID_ARG;
    int id = -1;
    for (int i = 0; i < K_COUNT; ++i)
        if (strcmp(name, kKernelNames[i]) == 0) id = i;
    if (id < 0) return SSD_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_timer_mu);
    double ms_sum = 0.0;
    int status = SSD_OK;
    for (auto &pr : g_timed[id]) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(pr.second);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
        if (e != cudaSuccess) status = cuda_status(e);
        ms_sum += ms;
        g_event_pool.push_back(pr.first);
        g_event_pool.push_back(pr.second);
    }
    if (total_ms) *total_ms = ms_sum;
    if (launches) *launches = (long long)g_timed[id].size();
    g_timed[id].clear();
    return status;
}

}  // extern "C"
