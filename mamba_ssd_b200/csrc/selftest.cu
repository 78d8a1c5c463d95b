// selftest.cu -- a self-test of the bounded waits of the tensor-core kernels.
//
// One warp waits, through the same bounded-wait helper the prefill kernels use, on an mbarrier
// that no thread ever arrives at.  The wait runs out after the given limit, records
// SSD_ERR_TIMEOUT in the status word and returns, so the failure path is exercised without
// faulting or hanging the GPU and the context stays usable afterwards.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace ssd {

__global__ void __launch_bounds__(32) selftest_wait_kernel(int *__restrict__ status, unsigned long long limit_ns) {
    using namespace tc;
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival, which never comes
        fence_barrier_init();
    }
    __syncwarp();
    mbar_wait(&bar, 0, status, limit_ns);
}

cudaError_t launch_selftest_wait(int *status, int limit_us, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(status, (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace ssd
