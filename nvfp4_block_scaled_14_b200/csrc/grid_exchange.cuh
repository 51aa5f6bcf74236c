// grid_exchange.cuh -- a bounded grid-wide barrier that also exchanges one pair of fp32
// maxima per CTA, for single-pass kernels whose CTAs are all resident at once (cooperative
// launch). The quantizers with a dynamic per-tensor amax use it: every CTA must have folded
// its share of the tensor before any CTA can compute the global scale.
//
// Values: each CTA writes its two maxima into its own 8-byte slot of the caller's workspace
// before it arrives (the workspace's earlier contents do not matter: every slot read after
// the barrier was written by this launch).
//
// Barrier: a sense-reversing counter (GridBarrier) in device memory that the library owns,
// zero when the library loads, and left with count 0 by every barrier that completes. A CTA
// reads the generation, arrives on the counter (release), and the last of the nblk CTAs to
// arrive resets the counter and advances the generation (release); the others poll the
// generation (acquire) for at most `limit` rounds. The host gives each stream its own
// GridBarrier and every launch captured into a CUDA graph a fresh one, so launches that may
// run at the same time never share one; launches on one stream are serialized, and each
// waits for its predecessor (programmatic dependent launch) before it touches the barrier.
// A barrier that ran out of rounds stays unbalanced until nvfp4_sync_status, which reports
// the timeout, resets the library's barriers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kExchangeMaxCtas = 160; // slots read per lane: 5

struct GridBarrier {
    uint32_t count; // arrivals of the barrier in progress
    uint32_t gen;   // completed barriers (wraps)
};

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrive on the barrier and wait (one thread per CTA). The relaxed read of gen comes before
// the arrival, whose release orders it (and this CTA's slot write) before any later arrival;
// gen cannot advance before this CTA has arrived. Returns false after `limit` poll rounds.
__device__ __forceinline__ bool grid_barrier_sync(GridBarrier *bar, int nblk, uint32_t limit)
{
    const uint32_t g0 = ld_relaxed_u32(&bar->gen);
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(&bar->count)
                 : "memory");
    if (old == (uint32_t)nblk - 1u) {
        // the last arrival: every other CTA's arrival (and what it released) is visible here
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(&bar->count) : "memory");
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&bar->gen), "r"(g0 + 1u)
                     : "memory");
        return true;
    }
    for (uint32_t round = 0; round < limit; ++round)
        if (ld_acquire_u32(&bar->gen) != g0)
            return true;
    return false;
}

// Called by all 32 lanes of one warp of each of the nblk (<= kExchangeMaxCtas) CTAs, with
// this CTA's values (va, vb: non-negative maxima; lane 0's are published). On return every
// lane holds the maxima over all CTAs in ga, gb. Returns false if the barrier ran out of
// rounds (ga, gb are then not meaningful).
__device__ __forceinline__ bool grid_exchange_max(float *slots, GridBarrier *bar, int nblk,
                                                  int bid, float va, float vb, uint32_t limit,
                                                  float &ga, float &gb)
{
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) {
        asm volatile("st.relaxed.gpu.global.v2.f32 [%0], {%1, %2};" ::"l"(slots + 2 * bid),
                     "f"(va), "f"(vb)
                     : "memory");
        ok = grid_barrier_sync(bar, nblk, limit) ? 1 : 0;
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    constexpr int NU = (kExchangeMaxCtas + 31) / 32;
    float a = 0.0f, b = 0.0f;
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        const int i = lane + 32 * u;
        if (i < nblk) {
            float x, y;
            asm volatile("ld.relaxed.gpu.global.v2.f32 {%0, %1}, [%2];"
                         : "=f"(x), "=f"(y)
                         : "l"(slots + 2 * i)
                         : "memory");
            a = fmaxf(a, x);
            b = fmaxf(b, y);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    }
    ga = a;
    gb = b;
    return ok != 0;
}

// Host side (api.cu): the GridBarrier a launch on stream s uses on the current device (null
// if the library's barriers cannot be reached), and the reset after a timeout.
GridBarrier *grid_barrier_for(cudaStream_t s);
cudaError_t reset_grid_barriers();

} // namespace nvfp4
