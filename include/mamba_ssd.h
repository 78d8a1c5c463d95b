/*
 * mamba_ssd.h -- C ABI of libmamba_ssd.so, the Mamba-2 state-space-duality (SSD)
 * selective scan for NVIDIA B200 (sm_100a): chunked prefill and the O(1) cached
 * decode step.
 *
 * Sources of the operations (page title and section):
 *   "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching for
 *   Inference" (abstract): diagonal per-head dynamics, fixed-size chunking, cached
 *   decode whose cost does not depend on the sequence length.
 *   The article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn), cited [blog §x.y]:
 *   §1.1 discretisation, chunking, decay mask L = tril(exp(segsum)); §1.2 the
 *   intra-chunk contraction; §2.1 the constant-size state h in R^{H x P x N} and the
 *   (kernel_size-1) conv cache; §2.2 the cache update (roll the conv window, set the
 *   newest slot; ssm = ssm * A_bar + B_bar * x); §3.2 / §4.1 decay and state in fp32.
 *
 * The mathematics every entry point implements, for batch b, head h, group
 * g = h / (H/G), token t:
 *   dt_t = clip(softplus(dt[b,t,h] + dt_bias[h]), dt_min, dt_max)
 *   h_t  = exp(dt_t * (-exp(A_log[h]))) * h_{t-1} + dt_t * x[b,t,h,:] (outer) B[b,t,g,:]
 *   y[b,t,h,:] = h_t C[b,t,g,:] + D[h] * x[b,t,h,:]
 * (the sign of A restored as -exp(A_log); B_bar = dt * B; y reads the state after
 * the update at t).
 *
 * Conventions shared by every call:
 *   - Every array argument is a DEVICE pointer owned by the caller.  The library
 *     never allocates device memory, never synchronises, and enqueues all of its
 *     work on `stream` (a cudaStream_t; NULL is the legacy default stream).  It
 *     returns as soon as the work is enqueued.
 *   - Arrays are dense, row-major, in exactly the index order written beside them.
 *     Every pointer must be 16-byte aligned.  Inputs are read-only unless marked
 *     "in/out".  Outputs must not alias inputs.
 *   - `dtype` selects the storage type of the activation arrays: SSD_DTYPE_F32
 *     (float) or SSD_DTYPE_BF16 (bfloat16).  Parameters and states (A_log, D,
 *     dt_bias, h0, h_final, ssm_state) are always float32.  Accumulation and the
 *     state recurrence are float32 in both cases.
 *   - Arguments are validated before anything is enqueued; on any error nothing is
 *     launched and an SSD_ERR_* code is returned.  A failed launch returns
 *     SSD_ERR_CUDA; the CUDA error code is kept per host thread
 *     (ssd_last_cuda_error) and a sticky CUDA error is not cleared.  No kernel traps.
 *   - The tensor-core prefill and the decode step are launched with programmatic
 *     dependent launch: a kernel may be scheduled while the one before it in the stream
 *     finishes, and reads and writes global memory only after that one has completed.
 *     The one exception is the decode state kernel's reads of ssm_state, which begin while
 *     the same call's conv kernel (which does not touch ssm_state) runs, but only after
 *     every kernel enqueued before the call has completed.  Setting SSD_PDL=0 in the environment (read once per process) launches them as
 *     ordinary kernels.
 *
 * Version 2: ssd_decode_status and ssd_selftest_wait_timeout added; the decode workspace
 * gained a status word (ssd_decode_workspace_size grew by 256 bytes).
 * Version 3: the decode step runs as two kernels; ssd_decode_workspace_size takes
 * (B, H, P, G, N), the workspace holds the step's conv outputs instead of arrival counters
 * and needs no zero-fill; the kernel timer knows "decode_conv"; ssd_gated_rmsnorm_fwd and
 * ssd_chunk_scan_varlen_fwd added.
 * Version 4: ssd_conv_chunk_scan_fwd / ssd_conv_chunk_scan_workspace_size (conv and prefill in
 * one call), ssd_segment_decay and ssd_state_combine (context-parallel prefill) added;
 * ssd_chunk_scan_fwd takes y = NULL (state only); ssd_chunk_scan_status(NULL) reads the
 * allocation-free entry's scratch.
 * Version 5: ssd_chunk_scan_varlen_fwd runs a packed batch in one pass on the tensor-core
 * path and takes its workspace size from the new ssd_chunk_scan_varlen_workspace_size.
 */
#ifndef MAMBA_SSD_H
#define MAMBA_SSD_H

#include <stddef.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-valued entry point. */
#define SSD_OK 0
#define SSD_ERR_INVALID_ARG 1  /* null/misaligned pointer, negative or inconsistent size */
#define SSD_ERR_UNSUPPORTED 2  /* valid request outside what the kernels implement */
#define SSD_ERR_WORKSPACE 3    /* workspace missing or smaller than the size query */
#define SSD_ERR_CUDA 4         /* a CUDA call or kernel launch failed */
#define SSD_ERR_TIMEOUT 5      /* a bounded device-side wait gave up */

/* Storage types of activation arrays. */
#define SSD_DTYPE_F32 0
#define SSD_DTYPE_BF16 1

/* Short English description of a status code (static storage, never NULL). */
SSD_API const char *ssd_status_string(int status);

/* The cudaError_t of the last SSD_ERR_CUDA returned on this host thread (0 if none). */
SSD_API int ssd_last_cuda_error(void);

/* Library ABI version, bumped on any signature change. */
SSD_API int ssd_abi_version(void);

/*
 * Bytes of device workspace that ssd_chunk_scan_fwd needs for this shape (a multiple
 * of 256; 0 when B == 0).  Returns 0 as well for shapes that
 * ssd_chunk_scan_fwd would reject.  Pure host computation.
 */
SSD_API size_t ssd_chunk_scan_workspace_size(int B, int L, int H, int P, int G, int N, int chunk,
                                     int dtype);

/*
 * Chunked SSD prefill ([blog §1.1, §1.2]; the state passing and the output
 * correction C h_prev exp(cumsum) + D x are the plain reading of §1.1):
 *   x        [B, L, H, P]  dtype      inputs
 *   dt       [B, L, H]     dtype      raw step sizes (before softplus, bias and clip)
 *   A_log    [H]           float      A = -exp(A_log)
 *   Bm, Cm   [B, L, G, N]  dtype      input and output projections of the state
 *   D        [H]           float      skip weight, NULL = 0
 *   dt_bias  [H]           float      NULL = 0
 *   dt_min, dt_max                    clip range of dt (0 and +inf disable it)
 *   h0       [B, H, P, N]  float      initial state, NULL = zeros
 *   y        [B, L, H, P]  dtype      output; NULL = only h_final is computed (the state the
 *                                      sequence leaves: the output kernels are skipped)
 *   h_final  [B, H, P, N]  float      state after token L-1 (h0 when L == 0); NULL = not written
 *   chunk                              tokens per chunk; the last chunk may be ragged
 *   workspace, workspace_bytes         >= ssd_chunk_scan_workspace_size(...), 256-byte
 *                                      aligned, contents on entry irrelevant; it is
 *                                      scratch for this call only, and after the call
 *                                      only its status word (ssd_chunk_scan_status) is
 *                                      defined: the tensor-core kernels drop the block
 *                                      states and h_prev from L2 once read, without
 *                                      writing them back
 * Supported: H % G == 0, P == 64, N in {16, 32, 64, 128}, chunk in {64, 128, 256, 512},
 * L >= 0, B >= 0.  Other valid shapes return SSD_ERR_UNSUPPORTED.  Calls sharing a
 * workspace must be ordered on one stream.
 * Kernels: bf16 storage with N == 128 runs on the tcgen05 tensor cores, which compute the
 * chunked form in 128-token blocks whatever `chunk` is (the decomposition is exact, only the
 * rounding differs); float32 storage and the other N run on float32 CUDA-core kernels with
 * the caller's chunk.  Setting SSD_PREFILL_KERNELS=simt in the environment (read once per
 * process) sends every shape to the CUDA-core kernels.
 */
SSD_API int ssd_chunk_scan_fwd(const void *x, const void *dt, const float *A_log, const void *Bm,
                       const void *Cm, const float *D, const float *dt_bias, float dt_min,
                       float dt_max, const float *h0, void *y, float *h_final, int B, int L,
                       int H, int P, int G, int N, int chunk, int dtype, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * The block step before the scan and the chunked prefill in one call: raw conv inputs in, the
 * scan's outputs and both caches out ([blog §2.1]: the depthwise sliding-window conv kept
 * beside the state, its (kernel_size - 1) input cache; [blog §1.1, §1.2]: the chunked scan;
 * [blog §3.2]: neighbouring element-wise work fused with the scan's data flow).
 *   xBC            [B, L, Cc]    dtype  raw conv inputs, channels [x | B | C], Cc = H*P + 2*G*N
 *   conv_w         [Cc, K]       dtype  depthwise taps, tap K-1 multiplies the newest input
 *   conv_b         [Cc]          dtype  conv bias, NULL = 0
 *   dt, A_log, D, dt_bias, dt_min, dt_max, h0, chunk, dtype   as for ssd_chunk_scan_fwd
 *   y              [B, L, H, P]  dtype  output of the scan over x, B, C = SiLU(conv(xBC) + b)
 *   h_final        [B, H, P, N]  float  NULL = not written
 *   conv_state_out [B, Cc, K-1]  dtype  the last K-1 raw inputs, oldest first, zeros before the
 *                                       start: with h_final, the cache ssd_decode_step continues
 *                                       from; NULL = not written
 *   workspace      >= ssd_conv_chunk_scan_workspace_size(...) bytes, 256-byte aligned
 * The workspace holds the prefill's scratch (first, so ssd_chunk_scan_status(workspace, ...)
 * reads this call's status) and then the conv output u [B, L, Cc]; the prefill kernels read
 * x, B and C as strided views of u (token rows Cc elements apart) right after the conv kernel
 * has written it, without splitting or copying it.  Supported: the shapes of
 * ssd_chunk_scan_fwd and of ssd_causal_conv1d_fwd (2 <= K <= 8, Cc % 8 == 0, B <= 65535).
 * Errors and ordering rules as for ssd_chunk_scan_fwd (everything checked before the first
 * launch).
 */
SSD_API size_t ssd_conv_chunk_scan_workspace_size(int B, int L, int H, int P, int G, int N, int K, int chunk,
                                                  int dtype);
SSD_API int ssd_conv_chunk_scan_fwd(const void *xBC, const void *conv_w, const void *conv_b, const void *dt,
                                    const float *A_log, const float *D, const float *dt_bias, float dt_min,
                                    float dt_max, const float *h0, void *y, float *h_final, void *conv_state_out,
                                    int B, int L, int H, int P, int G, int N, int K, int chunk, int dtype,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Context-parallel prefill: the sequence split into W consecutive segments, segment r on its
 * own GPU ([blog §1.1]: chunks computed in parallel, the state passed between them by a light
 * sequential scan; the segments are the chunks of that scan, one per GPU).  The recurrence is
 * linear in the state, so segment r maps its incoming state h_in to
 *   exp(sum_{t in segment} dt_t A) h_in + S_r,
 * with S_r the state it leaves when started from zero (ssd_chunk_scan_fwd with y = NULL and
 * h0 = NULL).  The steps per GPU: S_r and ssd_segment_decay; one all-gather of both over the
 * GPUs (NCCL, outside this library); ssd_state_combine for the segment's carry-in; then
 * ssd_chunk_scan_fwd over the segment from that carry-in (h0), which gives the segment's y.
 * ssd_state_combine with r = W gives the state after the whole sequence on every GPU.
 *
 * ssd_segment_decay: log2 of each (batch, head) segment's total decay,
 *   log2_decay[b, h] = -exp(A_log[h]) * sum_t clip(softplus(dt[b,t,h] + dt_bias[h]), dt_min, dt_max) * log2(e)
 *   dt [B, L, H] dtype (raw); A_log, dt_bias [H] float (dt_bias nullable); log2_decay [B, H] float.
 *   L = 0 gives 0.  Errors: SSD_ERR_INVALID_ARG for bad sizes, dtype, clip range or pointers.
 *
 * ssd_state_combine: the state entering segment r,
 *   h = h0 (or 0);  for j = 0 .. r-1:  h = exp2(log2_decays[j]) * h + states[j];  out = h
 *   states [r, B, H, P, N] float (the gathered S_j), log2_decays [r, B, H] float, h0 and out
 *   [B, H, P, N] float (h0 nullable; out must not overlap the inputs).  r = 0 copies h0 (or
 *   zeros).  Errors: SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED if P*N is not a multiple of 4.
 * Both are asynchronous on `stream` like every other entry point.
 */
SSD_API int ssd_segment_decay(const void *dt, const float *A_log, const float *dt_bias, float dt_min, float dt_max,
                              float *log2_decay, int B, int L, int H, int dtype, void *stream);
SSD_API int ssd_state_combine(const float *states, const float *log2_decays, const float *h0, float *out, int r,
                              int B, int H, int P, int N, void *stream);

/*
 * Varlen prefill: n_seq sequences of different lengths packed into one token stream, each
 * scanned on its own, as in the chunked prefill above ([blog §1.1]: the state is passed
 * along one sequence only).  Sequence i owns tokens cu_seqlens[i] .. cu_seqlens[i+1]-1:
 *   x [T, H, P], dt [T, H], Bm, Cm [T, G, N], y [T, H, P]   packed, T = cu_seqlens[n_seq]
 *   cu_seqlens  HOST array of n_seq + 1 ints, cu_seqlens[0] = 0, never decreasing (empty
 *               sequences allowed: their h_final is their h0, or 0)
 *   h0, h_final [n_seq, H, P, N] float, each nullable
 *   A_log, D, dt_bias, dt_min, dt_max, chunk, dtype   as for ssd_chunk_scan_fwd
 *   workspace   ssd_chunk_scan_varlen_workspace_size(cu_seqlens, n_seq, H, P, G, N, chunk,
 *               dtype) bytes, 256-byte aligned
 * On the tensor-core path (bf16, P = 64, N = 128) the batch runs in one pass: a small kernel
 * copies the table of its non-empty sequences (token start, first 128-token block, index)
 * from cu_seqlens into the workspace, then the three prefill kernels walk every (sequence,
 * block, head) item of the packed stream at once -- each sequence's blocks chained by the
 * state pass from its own h0 to its own h_final, the rows after a sequence's end masked out of
 * its last block -- so the launch count does not grow with n_seq.  An empty sequence's h_final
 * is copied from h0 (or zeroed) on `stream`.  On the CUDA-core path (and with
 * SSD_PREFILL_KERNELS=fused) each sequence runs the prefill kernels of ssd_chunk_scan_fwd with
 * B = 1, in order on `stream`, sharing the workspace.  Everything is validated before the first
 * launch: SSD_ERR_INVALID_ARG for bad cu_seqlens or pointers, SSD_ERR_UNSUPPORTED for a shape
 * ssd_chunk_scan_fwd would not take or, on the per-sequence path, a sequence whose dt rows
 * would not start 16-byte aligned (never when H * sizeof(element) is a multiple of 16),
 * SSD_ERR_WORKSPACE.  A CUDA launch error is returned as SSD_ERR_CUDA.  The workspace's status
 * word is this call's: ssd_chunk_scan_status reports SSD_ERR_TIMEOUT if any bounded wait of
 * the call gave up.
 *
 * ssd_chunk_scan_varlen_workspace_size: the bytes ssd_chunk_scan_varlen_fwd needs for this
 * batch (it grows with the total block count on the one-pass path), or 0 if n_seq <= 0 or an
 * argument is invalid.
 */
SSD_API size_t ssd_chunk_scan_varlen_workspace_size(const int *cu_seqlens, int n_seq, int H, int P, int G, int N,
                                                    int chunk, int dtype);
SSD_API int ssd_chunk_scan_varlen_fwd(const void *x, const void *dt, const float *A_log, const void *Bm,
                                      const void *Cm, const float *D, const float *dt_bias, float dt_min,
                                      float dt_max, const float *h0, void *y, float *h_final,
                                      const int *cu_seqlens, int n_seq, int H, int P, int G, int N, int chunk,
                                      int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Diagnostic: waits for `stream` to finish (this call synchronises, unlike every other
 * entry point) and returns the status the last ssd_chunk_scan_fwd on `workspace` left
 * there: SSD_OK, or SSD_ERR_TIMEOUT if one of its bounded device-side waits gave up (its
 * outputs are then incomplete).  A NULL workspace reads the built-in scratch of
 * ssd_chunk_scan_fwd_noalloc on the current device, i.e. the status of the last
 * allocation-free call there.  For ssd_chunk_scan_varlen_fwd it is the status of the whole
 * call: SSD_ERR_TIMEOUT if any of its kernels timed out.  SSD_ERR_CUDA if the stream,
 * the copy or the scratch lookup failed.
 */
SSD_API int ssd_chunk_scan_status(const void *workspace, void *stream);

/*
 * ssd_chunk_scan_fwd for callers that cannot allocate device memory.  (The paper and its
 * pages have no counterpart; this is an interface convenience of this library.)
 *
 * Who needs it: code that may not call cudaMalloc or any other allocating routine -- a
 * plugin inside a host engine that owns all device memory and forbids allocations after
 * start-up, a serving path that cannot afford the device synchronisation an allocation may
 * cause, or a runtime whose memory budget is fixed at load time -- but still has to run the
 * prefill, which needs scratch space.
 *
 * What it does: exactly ssd_chunk_scan_fwd (same arguments, same kernels, same results),
 * except that the scratch comes from one device array of SSD_NOALLOC_SCRATCH_BYTES compiled
 * into this library instead of a caller-provided workspace.  Every GPU on which the
 * library's device code is loaded holds that array until the process exits (see the lazy
 * loading note below for when that happens).  Inputs and outputs are still the caller's.
 *   - Shapes whose ssd_chunk_scan_workspace_size exceeds SSD_NOALLOC_SCRATCH_BYTES return
 *     SSD_ERR_WORKSPACE without launching anything (48 MiB covers, for example, one
 *     130M-shaped layer: batch 1, L = 4096, H = 24, P = 64, N = 128, bf16).
 *   - Every call looks up the array's device address on the current device (cheap once the
 *     library is loaded there; right across a device reset).  With lazy module loading, the
 *     CUDA default, the first call on a device also loads the library's device code there,
 *     and that is when the array's 48 MiB are committed on that device: make that first call
 *     at start-up, before any stream capture and before an engine reserves the rest of the
 *     device memory.  Later calls allocate nothing.
 *   - Its status word (SSD_ERR_TIMEOUT if a bounded device-side wait gave up) is read with
 *     ssd_chunk_scan_status(NULL, stream).
 *   - Every call uses the same array and leaves its contents behind.  Calls that may overlap
 *     on the GPU (different streams, different host threads without ordering) race on it and
 *     corrupt each other's results; order them on one stream.  Nothing in the array has to be
 *     zeroed by the caller.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine; the one commit of the
 *     array's memory is the driver's, when it loads the library's device code (above).
 */
#define SSD_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)
SSD_API int ssd_chunk_scan_fwd_noalloc(const void *x, const void *dt, const float *A_log,
                                       const void *Bm, const void *Cm, const float *D,
                                       const float *dt_bias, float dt_min, float dt_max,
                                       const float *h0, void *y, float *h_final, int B, int L,
                                       int H, int P, int G, int N, int chunk, int dtype,
                                       void *stream);

/*
 * Bytes of device workspace that ssd_decode_step needs (a multiple of 256); 0 if an
 * argument is not positive.  The workspace holds a status word, the step's conv outputs
 * (B * (H*P + 2*G*N) floats) and its (dt, exp(dt*A)) pairs (B * H float2).  It needs no
 * initialisation: every call writes what it reads.  One workspace serves any number of
 * calls of the same or smaller shape that are ordered on one stream.
 */
SSD_API size_t ssd_decode_workspace_size(int B, int H, int P, int G, int N);

/*
 * Diagnostic: synchronises `stream` and returns the status word the last ssd_decode_step
 * on `workspace` left; SSD_ERR_INVALID_ARG for a NULL workspace, SSD_ERR_CUDA if the stream
 * reported an error.  The decode kernels have no waits and always leave SSD_OK; the word is
 * there so that a kernel with bounded waits can report SSD_ERR_TIMEOUT without an ABI change.
 */
SSD_API int ssd_decode_status(const void *workspace, void *stream);

/*
 * One cached decode step for one layer ([blog §2.1, §2.2]), enqueued as two kernels on
 * `stream` (the conv and conv-cache roll, then the state update):
 *   ssm_state  [B, H, P, N]   float  in/out: h <- exp(dt*A) h + dt x (outer) B
 *   conv_state [B, Cc, K-1]   dtype  in/out: the K-1 most recent raw xBC inputs,
 *                                    oldest first; rolled by one and the newest input
 *                                    appended
 *   xBC_t      [B, Cc]        dtype  this token's raw conv input, channels [x | B | C],
 *                                    Cc = H*P + 2*G*N
 *   dt_t       [B, H]         dtype  raw step size
 *   A_log, D, dt_bias, dt_min, dt_max   as for ssd_chunk_scan_fwd (D, dt_bias nullable)
 *   conv_w     [Cc, K]        dtype  depthwise conv taps, tap K-1 multiplies the newest input
 *   conv_b     [Cc]           dtype  conv bias, NULL = 0
 *   y_t        [B, H, P]      dtype  output: y = h C + D x, with x, B, C = SiLU(conv + bias)
 *   workspace  ssd_decode_workspace_size(B, H, P, G, N) bytes, 16-byte aligned
 * Supported: H % G == 0, P % 16 == 0, N in {16, 32, 64, 128, 256}, 2 <= K <= 8,
 * B <= 65535 (else SSD_ERR_UNSUPPORTED).  Calls sharing a workspace must be ordered on one
 * stream.  With programmatic dependent launch (below), the state kernel starts reading
 * ssm_state while the step's own conv kernel runs, after every kernel enqueued before the
 * call has completed: ssm_state must not be written by anything running concurrently with
 * the call, the same rule as for any other argument.
 */
SSD_API int ssd_decode_step(float *ssm_state, void *conv_state, const void *xBC_t, const void *dt_t,
                    const float *A_log, const float *D, const float *dt_bias, float dt_min,
                    float dt_max, const void *conv_w, const void *conv_b, void *y_t, int B,
                    int H, int P, int G, int N, int K, int dtype, void *workspace,
                    size_t workspace_bytes, void *stream);

/*
 * Causal depthwise conv1d + bias + SiLU over a prefix, zero left padding ([blog §2.1]
 * sliding-window conv), and the conv cache it leaves for decode:
 *   xBC            [B, L, Cc]  dtype  raw inputs
 *   conv_w         [Cc, K]     dtype  tap K-1 multiplies the newest input
 *   conv_b         [Cc]        dtype  NULL = 0
 *   out            [B, L, Cc]  dtype  SiLU(sum_k w[c,k] xBC[t-K+1+k, c] + b[c])
 *   conv_state_out [B, Cc, K-1] dtype the last K-1 raw inputs, oldest first, zeros
 *                                     before the start; NULL = not written
 * Supported: 2 <= K <= 8, Cc % 8 == 0, 0 <= L <= 2097120, B <= 65535.  Launched with
 * programmatic dependent launch.
 */
SSD_API int ssd_causal_conv1d_fwd(const void *xBC, const void *conv_w, const void *conv_b, void *out,
                          void *conv_state_out, int B, int L, int Cc, int K, int dtype,
                          void *stream);

/*
 * Gated RMS norm, the block step after the scan ([blog §4.1]: a norm takes its variance in
 * float32 even for bf16 inputs; the gate and the per-group RMS are the Mamba-2 block's norm,
 * which the pages name without spelling out):
 *   g   = y * SiLU(z)
 *   out = g / sqrt(mean over the channels of its group of g^2 + eps) * w
 *   y, z  [T, C]  dtype  the scan output and the gate input, T tokens of C channels (for a
 *                        prefill output y[B, L, H, P]: T = B*L, C = H*P)
 *   w     [C]     float  per-channel scale
 *   out   [T, C]  dtype  must not overlap y or z
 *   n_groups             norm groups per token: C / n_groups consecutive channels each
 * The mean square is accumulated in float32.  The gate's exponential and division use the
 * GPU's approximate instructions (relative error about 2^-21), and so does the reciprocal
 * square root for groups of up to 10240 bf16 / 5120 float32 channels.
 * Supported: C % n_groups == 0,
 * C / n_groups a multiple of 8 and at most 32768, n_groups <= 65535, eps >= 0 and finite.
 * Pointers 16-byte aligned.  Errors: SSD_ERR_INVALID_ARG (bad sizes, eps, dtype, pointers),
 * SSD_ERR_UNSUPPORTED (group size), SSD_ERR_CUDA.  T == 0 is a no-op.  Launched with
 * programmatic dependent launch like the prefill kernels.
 */
SSD_API int ssd_gated_rmsnorm_fwd(const void *y, const void *z, const float *w, void *out, int T, int C,
                                  int n_groups, float eps, int dtype, void *stream);

/*
 * Self-test of the bounded waits (no counterpart in the pages; the failure path of the
 * tensor-core kernels).  Launches one warp that waits, with the same bounded-wait code the
 * prefill kernels use, on an mbarrier that no thread ever arrives at, giving up after
 * `limit_us` microseconds (1 .. 1000000).  It then stores SSD_ERR_TIMEOUT into `status` (one
 * device int, caller-owned) and returns; nothing faults or hangs and the context stays
 * usable.  Returns SSD_ERR_INVALID_ARG for a NULL or misaligned status or a limit out of
 * range, SSD_ERR_CUDA if the launch failed, else SSD_OK (asynchronous on `stream`).
 */
SSD_API int ssd_selftest_wait_timeout(int *status, int limit_us, void *stream);

/*
 * Profiling hooks (host-side bookkeeping; no device memory is allocated).
 *
 * ssd_kernel_launch_count: kernels this library has enqueued in this process so far
 * (every entry point, every host thread).
 *
 * ssd_kernel_timer_enable(1) makes every later kernel launch on this process record a
 * pair of CUDA events around itself on its own stream; ssd_kernel_timer_read(name, ...)
 * waits for the recorded events of kernel `name` ("decay_prep", "chunk_state",
 * "state_pass", "chunk_scan", "run_state", "run_pass", "chunk_scan_fused", "decode_conv",
 * "decode_step" (the decode state update), "causal_conv1d", "gated_rmsnorm", "segment_decay",
 * "state_combine"), returns the summed
 * device time in milliseconds and the number of launches timed, and forgets them.
 * Do not enable the timer while a stream is being captured into a CUDA graph.
 * Returns SSD_OK, SSD_ERR_INVALID_ARG for an unknown name, SSD_ERR_CUDA on an event error.
 */
SSD_API long long ssd_kernel_launch_count(void);
SSD_API int ssd_kernel_timer_enable(int on);
SSD_API int ssd_kernel_timer_read(const char *name, double *total_ms, long long *launches);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_SSD_H */
