// noalloc.cu -- ssd_chunk_scan_fwd_noalloc: the chunked SSD prefill for callers that cannot
// allocate device memory.
//
// Some callers are not allowed to call cudaMalloc or any other allocating routine: a plugin
// inside a host inference engine that owns all device memory and forbids allocations after
// start-up, a real-time serving path that cannot afford the implicit device synchronisation
// an allocation can cause, or a runtime with a fixed memory budget decided at load time.
// They still need the prefill's scratch space (per-token decay data and per-chunk states).
// This entry point takes it from one file-scope device array, sized at compile time, that
// every GPU loading this library holds until the process exits.
//
// The kernels, their launch order and their results are exactly those of
// ssd_chunk_scan_fwd; only the scratch pointer differs.
#include "common.cuh"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = SSD_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// The shared scratch.  In host code `g_noalloc_scratch` names a host-side stand-in, not the
// device array: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

}  // namespace

namespace ssd {
// Device address of the scratch array on the current device, looked up on every call: it is
// cheap once the library's module is loaded, and stays right across a device reset, which
// reloads the module (possibly at another address).  With lazy module loading (the CUDA
// default) the first lookup on a device loads the module, which is when the array's memory
// is committed on that device.
cudaError_t noalloc_scratch(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}
}  // namespace ssd

extern "C" int ssd_chunk_scan_fwd_noalloc(const void *x, const void *dt, const float *A_log,
                                          const void *Bm, const void *Cm, const float *D,
                                          const float *dt_bias, float dt_min, float dt_max,
                                          const float *h0, void *y, float *h_final, int B, int L,
                                          int H, int P, int G, int N, int chunk, int dtype,
                                          void *stream) {
    // shape checks first, so that an oversized request fails before any CUDA call
    const size_t need = ssd_chunk_scan_workspace_size(B, L, H, P, G, N, chunk, dtype);
    if (need > kScratchBytes) return SSD_ERR_WORKSPACE;
    if (B > 0 && need == 0 && L > 0)  // shape rejected by the size query: let the call say why
        return ssd_chunk_scan_fwd(x, dt, A_log, Bm, Cm, D, dt_bias, dt_min, dt_max, h0, y, h_final, B,
                                  L, H, P, G, N, chunk, dtype, nullptr, 0, stream);
    void *scratch = nullptr;
    const cudaError_t e = ssd::noalloc_scratch(&scratch);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    // Nothing in the scratch has to start at zero: the prefill overwrites every byte it reads
    // (its status word is reset by the call's first kernel).
    return ssd_chunk_scan_fwd(x, dt, A_log, Bm, Cm, D, dt_bias, dt_min, dt_max, h0, y, h_final, B, L,
                              H, P, G, N, chunk, dtype, scratch, kScratchBytes, stream);
}
