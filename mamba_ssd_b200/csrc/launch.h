// launch.h -- internal launchers of the SSD kernels (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ssd {

// Prefill workspace layout, 256-byte aligned pieces:
//   status int32 (256-byte slot): SSD_OK, or SSD_ERR_TIMEOUT if a bounded wait gave up
//   dtf    [B][H][Lp]          clipped dt per token (0 past the end of the sequence)
//   acs    [B][H][Lp]          inclusive cumsum of dt*A inside each chunk
//   states [B][nc][H][P][N]    chunk states, overwritten in place by the state each
//                              chunk starts from (h_prev)
// with nc = ceil(L / chunk), Lp = nc * chunk.
struct PrefillWorkspace {
    int *status;
    float *dtf;
    float *acs;
    float *states;
};
size_t prefill_workspace_bytes(int B, int L, int H, int P, int N, int chunk);
PrefillWorkspace carve_prefill_workspace(void *base, int B, int L, int H, int P, int N, int chunk);

cudaError_t launch_decay_prep(int dtype, const void *dt, const float *A_log, const float *dt_bias,
                              float dt_min, float dt_max, float *dtf, float *acs, int *status, int B,
                              int L, int H, int chunk, cudaStream_t st);

// tensor-core chunk state (bf16 storage, P = 64, N = 128, chunk 256)
bool chunk_state_tc_supported(int dtype, int P, int N, int chunk);
cudaError_t launch_chunk_state_tc(const void *x, const void *Bm, const float *dtf, const float *acs,
                                  float *states, int *status, int B, int L, int H, int G,
                                  int num_sms, cudaStream_t st);

// tensor-core chunk scan (bf16 storage, P = 64, N = 128, chunk 256)
bool chunk_scan_tc_supported(int dtype, int P, int N, int chunk);
cudaError_t launch_chunk_scan_tc(const void *x, const void *Bm, const void *Cm, const float *dtf,
                                 const float *acs, const float *hprev, const float *D, void *y,
                                 int *status, int B, int L, int H, int G, int num_sms, cudaStream_t st);

cudaError_t launch_chunk_state(int dtype, const void *x, const void *Bm, const float *dtf,
                               const float *acs, float *states, int B, int L, int H, int G, int N,
                               int chunk, cudaStream_t st);

cudaError_t launch_state_pass(float *states, const float *acs, const float *h0, float *h_final,
                              int B, int L, int H, int P, int N, int chunk, cudaStream_t st);

cudaError_t launch_chunk_scan(int dtype, const void *x, const void *Bm, const void *Cm,
                              const float *dtf, const float *acs, const float *hprev,
                              const float *D, void *y, int B, int L, int H, int G, int N,
                              int chunk, cudaStream_t st);

cudaError_t launch_decode_step(int dtype, float *ssm_state, void *conv_state, const void *xBC_t,
                               const void *dt_t, const float *A_log, const float *D,
                               const float *dt_bias, float dt_min, float dt_max,
                               const void *conv_w, const void *conv_b, void *y_t, int B, int H,
                               int P, int G, int N, int K, unsigned *counters, cudaStream_t st);

cudaError_t launch_causal_conv1d(int dtype, const void *xBC, const void *conv_w,
                                 const void *conv_b, void *out, void *conv_state_out, int B,
                                 int L, int Cc, int K, cudaStream_t st);

}  // namespace ssd
