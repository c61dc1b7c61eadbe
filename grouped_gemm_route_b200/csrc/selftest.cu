// Self-test of the device-side failure path: a kernel waits, with the same
// bounded mbarrier wait the GEMM pipelines use, on a barrier that nothing
// arrives at.  The wait expires after the time limit and the kernel records a
// timeout in the status word and returns; nothing is left in flight, so the
// context stays usable.
#include <cuda_runtime.h>

#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

__global__ void expire_wait_kernel(int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0u, nullptr)) report_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_expire_wait(int *status, cudaStream_t s) {
    expire_wait_kernel<<<1, 32, 0, s>>>(status);
    return cudaGetLastError();
}

}  // namespace moe
