// varlen.cu -- the table a packed varlen prefill runs from (items.cuh, struct Varlen).
//
// The caller's cumulative lengths are a host array; the tensor-core kernels walk the packed
// batch's (sequence, block, head) items from a copy of its non-empty sequences in the
// workspace.  This kernel writes that copy from its launch parameters (a kernel launch, not a
// host-to-device copy, so the call stays capturable into a CUDA graph from pageable host
// memory); a batch with more sequences than one launch carries is written in several.
#include "common.cuh"
#include "launch.h"

namespace ssd {

__global__ void __launch_bounds__(256) varlen_table_kernel(const VarlenTableChunk c, int *__restrict__ tok0,
                                                           int *__restrict__ blk0, int *__restrict__ seq) {
    grid_dependency_wait();  // the workspace may still be read by the kernels before this call
    allow_dependents();
    tok0 = after_wait(tok0);
    blk0 = after_wait(blk0);
    seq = after_wait(seq);
    for (int i = threadIdx.x; i < c.count; i += blockDim.x) {
        tok0[c.base + i] = c.tok0[i];
        blk0[c.base + i] = c.blk0[i];
        seq[c.base + i] = c.seq[i];
    }
}

cudaError_t launch_varlen_table(const VarlenTableChunk &c, int *tok0, int *blk0, int *seq, cudaStream_t st) {
    return launch_pdl(varlen_table_kernel, dim3(1), dim3(256), 0, st, c, tok0, blk0, seq);
}

}  // namespace ssd
