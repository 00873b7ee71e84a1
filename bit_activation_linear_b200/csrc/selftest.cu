// selftest.cu -- exercises the library's failure detection without faulting or hanging the GPU.
//
// Every wait in the library's kernels is bounded (mbar_wait): when a phase does not complete in
// time the kernel records BITNET_ERR_TIMEOUT in the device status word, winds down and returns,
// and bitnet_sync_status() reports it.  This kernel runs that same bounded wait on an mbarrier no
// thread ever arrives on, with a short limit, so the whole path can be checked on a healthy GPU.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

__global__ void selftest_wait_timeout_kernel(long long limit_cycles, int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival would complete phase 0; none is ever made
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, status, limit_cycles);
}

cudaError_t launch_selftest_wait_timeout(long long limit_cycles, int *status,
                                         cudaStream_t stream) {
    selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_cycles, status);
    return cudaGetLastError();
}

}  // namespace bitnet
