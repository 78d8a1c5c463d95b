// launch.h -- internal launchers of the SSD kernels (not part of the public C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "items.cuh"
#include "runs.cuh"

namespace ssd {

// A kernel's dynamic shared-memory limit, raised once per device (the attribute is per device;
// raising it on every launch would cost a driver call each time).
template <auto Kernel>
cudaError_t raise_smem_limit(int bytes) {
    static std::atomic<unsigned long long> done{0};  // bit d: raised on device d
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// A kernel as a type, for generic lambdas that launch one of several instantiations.
template <auto K>
struct KernelTag {
    static constexpr auto kernel = K;
};

// Launches of the tensor-core prefill kernels use programmatic stream serialization (each may
// be scheduled while the kernel before it finishes; the kernels order every global access
// after griddepcontrol.wait).  SSD_PDL=0 in the environment turns it off.
bool pdl_enabled();
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Prefill workspace layout, 256-byte aligned pieces:
//   status int32 (256-byte slot): SSD_OK, or SSD_ERR_TIMEOUT if a bounded wait gave up
//   dtf    [B][H][Lp]          clipped dt per token (0 past the end of the sequence); on the
//                              tensor-core path its base-2 logarithm, log2(dt), instead, as
//                              [H][B*nb][128] (each head's blocks of the whole batch in a row)
//   acs    [B][H][Lp]          inclusive cumsum of dt*A inside each block; on the tensor-core
//                              path acs2 = that cumsum times log2(e), laid out like dtf
//   states [B][nb][H][P][N]    fp32 block states; the CUDA-core path overwrites them in
//                              place with the state each block starts from (h_prev); the
//                              tensor-core path stores each transposed, [N][P]
//   hT     [B][nb][H][N][P]    (tensor-core path) h_prev of each block, bf16, transposed
// with nb = ceil(L / block), Lp = nb * block.  The block is the caller's chunk on the
// CUDA-core path and 128 tokens (the tcgen05 M) on the tensor-core path.
struct PrefillWorkspace {
    int *status;
    float *dtf;
    float *acs;
    float *states;
    __nv_bfloat16 *hT;
};
size_t prefill_workspace_bytes(int B, int L, int H, int P, int N, int block, bool transposed_bf16);
PrefillWorkspace carve_prefill_workspace(void *base, int B, int L, int H, int P, int N, int block,
                                         bool transposed_bf16);

// Step a1 for the CUDA-core path: writes dt and acs (natural form) and resets the status word
// (when status is not NULL).
cudaError_t launch_decay_prep(int dtype, const void *dt, const float *A_log, const float *dt_bias,
                              float dt_min, float dt_max, float *dtf, float *acs, int *status, int B,
                              int L, int H, int chunk, cudaStream_t st);

// tensor-core prefill (bf16 storage, P = 64, N = 128), 128-token blocks
constexpr int kTcBlock = 128;
bool prefill_tc_supported(int dtype, int P, int N);
// chunk_state_tc also forms the log2-form decay factors (dtf = log2(dt), acs = acs2) from dt and
// resets the status word: it is the first kernel of a tensor-core prefill call.
// Their workspace (global block gb, head h: factor rows at (h*nblocks + gb)*128, states at
// (gb*H + h)*P*N), for an equal-length batch (B sequences of L tokens, nblocks = B*ceil(L/128),
// vl.n = 0) or a packed varlen batch (B = 1, L = the packed token count, vl = the non-empty
// sequences' table, nblocks = its block count).
cudaError_t launch_chunk_state_tc(const void *x, const void *Bm, const void *dt, const float *A_log,
                                  const float *dt_bias, float dt_min, float dt_max, float *dtf, float *acs,
                                  float *states, int *status, bool reset_status, int B, int L, int H, int G,
                                  int64_t x_row, int64_t bc_row, const Varlen &vl, int nblocks, int num_sms,
                                  cudaStream_t st);

cudaError_t launch_chunk_scan_tc(const void *x, const void *Bm, const void *Cm, const float *dtf,
                                 const float *acs, const __nv_bfloat16 *hT, const float *D, void *y,
                                 int *status, int B, int L, int H, int G, int64_t x_row, int64_t bc_row,
                                 const Varlen &vl, int nblocks, int num_sms, cudaStream_t st);
cudaError_t launch_state_pass_t(const float *states, const float *acs, const float *h0, float *h_final,
                                __nv_bfloat16 *hT, int B, int L, int H, int P, int N, int chunk, const Varlen &vl,
                                int nblocks, cudaStream_t st);

// Up to kVarlenChunk entries of a packed varlen batch's table, written at [base, base + count)
// of the workspace copy by one launch.
constexpr int kVarlenChunk = 256;
struct VarlenTableChunk {
    int base, count;
    int tok0[kVarlenChunk + 1], blk0[kVarlenChunk + 1], seq[kVarlenChunk + 1];
};
cudaError_t launch_varlen_table(const VarlenTableChunk &c, int *tok0, int *blk0, int *seq, cudaStream_t st);

// Fused tensor-core prefill (bf16 storage, P = 64, N = 128, an even number of heads per
// group): the work is split into runs of blocks per head pair (runs.cuh); three launches:
//   run_state_tc      each run's own state (hi/lo accurate) and total decay, into its slot;
//                     resets the status word (the first kernel of the call)
//   run_pass          the pass over each chain's runs: carry-ins in place of the run states,
//                     and h_final
//   chunk_scan_fused  y, with each head's state carried through its runs in TMEM
// Workspace: status (256-byte slot), then slots [lay.slots()][2][N][P] fp32, then decays
// [lay.slots()][2] fp32 (log2 of each run's total decay), each piece 256-byte aligned.
bool prefill_fused_supported(int dtype, int P, int N, int H, int G);
struct FusedWorkspace {
    int *status;
    float *slots;
    float *decays;
};
RunLayout fused_layout(int B, int L, int H, int num_sms);
size_t fused_workspace_bytes(int B, int L, int H);
FusedWorkspace carve_fused_workspace(void *base, int B, int L, int H);
cudaError_t launch_run_state_tc(const void *x, const void *Bm, const void *dt, const float *A_log,
                                const float *dt_bias, float dt_min, float dt_max, float *slots, float *decays,
                                int *status, bool reset_status, int B, int L, int H, int G, int64_t x_row,
                                int64_t bc_row, const RunLayout &lay, cudaStream_t st);
cudaError_t launch_run_pass(float *slots, const float *decays, const float *h0, float *h_final, int B, int H,
                            const RunLayout &lay, cudaStream_t st);
cudaError_t launch_chunk_scan_fused(const void *x, const void *Bm, const void *Cm, const void *dt, const float *A_log,
                                    const float *dt_bias, float dt_min, float dt_max, const float *D,
                                    const float *slots, void *y, int *status, int B, int L, int H, int G,
                                    int64_t x_row, int64_t bc_row, const RunLayout &lay, cudaStream_t st);

// x rows (tokens) are x_row elements apart and B/C rows bc_row apart: H*P and G*N when dense,
// wider when x, B and C are strided views into one [.., H*P + 2*G*N] conv output.
cudaError_t launch_chunk_state(int dtype, const void *x, const void *Bm, const float *dtf,
                               const float *acs, float *states, int B, int L, int H, int G, int N,
                               int chunk, int64_t x_row, int64_t bc_row, cudaStream_t st);

cudaError_t launch_state_pass(float *states, const float *acs, const float *h0, float *h_final,
                              int B, int L, int H, int P, int N, int chunk, cudaStream_t st);

cudaError_t launch_chunk_scan(int dtype, const void *x, const void *Bm, const void *Cm,
                              const float *dtf, const float *acs, const float *hprev,
                              const float *D, void *y, int B, int L, int H, int G, int N,
                              int chunk, int64_t x_row, int64_t bc_row, cudaStream_t st);

// One decode step is two launches: the conv kernel (conv, SiLU, conv-cache roll, dt and the
// decay factor, into u_ws [B][Cc] fp32 and da_ws [B][H] (dt, a)), then the state kernel.
cudaError_t launch_decode_conv(int dtype, void *conv_state, const void *xBC_t, const void *dt_t,
                               const float *A_log, const float *dt_bias, float dt_min, float dt_max,
                               const void *conv_w, const void *conv_b, float *u_ws, float2 *da_ws,
                               int B, int H, int P, int G, int N, int K, cudaStream_t st);

cudaError_t launch_decode_state(int dtype, float *ssm_state, const float *u_ws, const float2 *da_ws,
                                const float *D, void *y_t, int B, int H, int P, int G, int N, int *status,
                                cudaStream_t st);

// Gated RMS norm over T_rows tokens of C channels in n_groups groups (C / n_groups channels
// each, a multiple of the 16-byte vector and at most 32768).
cudaError_t launch_gated_rmsnorm(int dtype, const void *y, const void *z, const float *w, void *out, int T_rows,
                                 int C, int n_groups, float eps, cudaStream_t st);

cudaError_t launch_causal_conv1d(int dtype, const void *xBC, const void *conv_w,
                                 const void *conv_b, void *out, void *conv_state_out, int B,
                                 int L, int Cc, int K, cudaStream_t st);

// Context-parallel steps: each (batch, head) segment's total decay, log2 form, into out [B][H];
// and the carry-in h = h0 (or 0), h = exp2(ld_j) h + S_j for j < r, of [B][H][P][N] states.
cudaError_t launch_segment_decay(int dtype, const void *dt, const float *A_log, const float *dt_bias, float dt_min,
                                 float dt_max, float *out, int B, int L, int H, cudaStream_t st);
cudaError_t launch_state_combine(const float *states, const float *log2_decays, const float *h0, float *out, int r,
                                 int B, int H, int P, int N, cudaStream_t st);

// Device address, on the current device, of the built-in scratch array of
// ssd_chunk_scan_fwd_noalloc (its first 256 bytes hold that entry's status word).
cudaError_t noalloc_scratch(void **out);

// One warp waits on an mbarrier that nothing arrives at, for limit_us microseconds, and records
// SSD_ERR_TIMEOUT in *status (the bounded-wait self-test).
cudaError_t launch_selftest_wait(int *status, int limit_us, cudaStream_t st);

}  // namespace ssd
