// grid_exchange.cuh -- a bounded grid-wide barrier that also exchanges one pair of fp32
// maxima per CTA, for single-pass kernels whose CTAs are all resident at once (cooperative
// launch). The quantizers with a dynamic per-tensor amax use it: every CTA must have folded
// its share of the tensor before any CTA can compute the global scale.
//
// Values: each CTA writes its two maxima into its own 8-byte slot of the caller's workspace
// before it arrives (the workspace's earlier contents do not matter: every slot read after
// the barrier was written by this launch).
//
// Barrier: a counter word (GridBarrier) in device memory that the library owns, zero when the
// library loads. Each CTA adds to it once (release): CTA 0 adds 2^31 - (nblk - 1), the others
// 1, so bit 31 flips exactly when the last CTA arrives and the low bits return to zero (the
// state the next barrier needs); every CTA polls (acquire) for the flip against the value its
// own addition returned, for at most `limit` rounds. The host gives each stream its own
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
    uint32_t count; // bit 31: flips once per completed barrier; bits 0-30: arrivals so far
    uint32_t unused;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrive on the barrier and wait (one thread per CTA; bid: this CTA's index among the nblk).
// The arrival's release orders this CTA's slot write before it; the additions form one release
// sequence, so the poll that sees the flip (acquire) sees every CTA's slot. Returns false after
// `limit` poll rounds.
__device__ __forceinline__ bool grid_barrier_sync(GridBarrier *bar, int nblk, int bid,
                                                  uint32_t limit)
{
    const uint32_t add = bid == 0 ? 0x80000000u - (uint32_t)(nblk - 1) : 1u;
    uint32_t old;
    asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(&bar->count), "r"(add)
                 : "memory");
    for (uint32_t round = 0; round < limit; ++round)
        if (((ld_acquire_u32(&bar->count) ^ old) & 0x80000000u) != 0u)
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
        ok = grid_barrier_sync(bar, nblk, bid, limit) ? 1 : 0;
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
