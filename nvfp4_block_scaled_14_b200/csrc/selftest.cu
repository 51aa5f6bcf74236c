// selftest.cu -- exercises the library's device-side timeout path without a GPU fault.
//
// Every wait in the library's kernels is bounded: when it gives up, the kernel writes
// NVFP4_ERR_TIMEOUT into the library's status word, finishes without the missing data and
// returns, and nvfp4_sync_status reports the status. This kernel takes that path on purpose:
// it waits on an mbarrier that nothing arrives on, with a short poll limit. A second kernel
// runs the quantizers' bounded grid-wide exchange on its own, with one CTA that may stay away
// (its peers' barrier then runs out) and one that may arrive late (its peers must wait for it,
// whatever earlier launches left in the workspace).
#include "grid_exchange.cuh"
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

// Every CTA but `skip` exchanges (vals[bid], vals[bid] / 2) with grid_exchange_max; CTA `late`
// first spins for late_ns nanoseconds. CTA 0 writes the maxima to out[0..1]; an exchange that
// runs out of its `limit` poll rounds records NVFP4_ERR_TIMEOUT and returns.
__global__ void exchange_selftest_kernel(float *slots, GridBarrier *bar, const float *vals,
                                         int skip, int late, uint32_t late_ns, uint32_t limit,
                                         float *out, int *status)
{
    const int bid = (int)blockIdx.x;
    if (bid == skip)
        return;
    if (bid == late && threadIdx.x == 0) {
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        do {
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        } while (t - t0 < late_ns);
    }
    __syncwarp();
    float ga, gb;
    const float v = vals[bid];
    const bool ok =
        grid_exchange_max(slots, bar, (int)gridDim.x, bid, v, 0.5f * v, limit, ga, gb);
    if (threadIdx.x == 0) {
        if (!ok)
            atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
        else if (bid == 0) {
            out[0] = ga;
            out[1] = gb;
        }
    }
}

} // namespace

cudaError_t launch_exchange_selftest(int nblk, const float *vals, int skip, int late,
                                     uint32_t late_ns, uint32_t limit, float *out, void *ws,
                                     cudaStream_t s)
{
    int *status = device_status_ptr();
    GridBarrier *bar = grid_barrier_for(s);
    if (!status || !bar)
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t c{};
    c.gridDim = dim3((unsigned)nblk);
    c.blockDim = dim3(32);
    c.stream = s;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeCooperative; // every CTA resident, as in the quantizers
    a[0].val.cooperative = 1;
    c.attrs = a;
    c.numAttrs = 1;
    return cudaLaunchKernelEx(&c, exchange_selftest_kernel, reinterpret_cast<float *>(ws), bar,
                              vals, skip, late, late_ns, limit, out, status);
}

cudaError_t launch_wait_timeout_selftest(cudaStream_t s)
{
    int *status = device_status_ptr();
    if (!status)
        return cudaErrorInvalidValue;
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, 256u);
    return cudaGetLastError();
}

} // namespace nvfp4
