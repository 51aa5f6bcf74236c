// selftest.cu -- exercises the library's device-side timeout path without a GPU fault.
//
// Every wait in the library's kernels is bounded: when it gives up, the kernel writes
// NVFP4_ERR_TIMEOUT into the library's status word, finishes without the missing data and
// returns, and nvfp4_sync_status reports the status. This kernel takes that path on purpose:
// it waits on an mbarrier that nothing arrives on, with a short poll limit.
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

__global__ void wait_timeout_kernel(int *status, uint32_t limit)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit)) // phase 0 never completes
        atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
}

} // namespace

cudaError_t launch_wait_timeout_selftest(cudaStream_t s)
{
    int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidValue;
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, 256u);
    return cudaGetLastError();
}

} // namespace nvfp4
