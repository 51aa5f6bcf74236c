// calib.cu -- exact nearest-rank percentile of |x| (and max |x|) over a set of device
// batches, for static NVFP4 input scales ("Qwen-Rapid-AIO FP8 -> NVFP4", "Recommended
// Model": p99.9 percentile aggregation over calibration generations instead of max).
//
// |x| orders like its bit pattern with the sign cleared, so the rank-th smallest |x| is found
// by counting bit patterns:
//   bf16: one pass. A 32768-bin histogram of the 15 magnitude bits is exact.
//   fp32: two passes. Pass 1 bins the high 15 magnitude bits; the bin holding the rank is
//         then resolved by a 65536-bin histogram of the low 16 bits of the values inside it.
// Each CTA keeps a private 128 KB shared-memory histogram (one CTA per SM), adds it to the
// global 64-bit histogram once, and folds max |x| into one word with atomicMax on the bits.
// A single-CTA select kernel scans the histogram on the device, so no host sync is needed
// and the result is independent of the order in which CTAs run.
#include "nvfp4_internal.cuh"

namespace nvfp4 {
namespace {

constexpr int kHistThreads = 1024;
constexpr int kBins1 = 32768;
constexpr int kBins2 = 65536;
constexpr int kMaxBatchesPerLaunch = 64;
// 16-byte loads in flight per thread (measured 4 / 8 / 16 on B200: 4 or 8 best; the pass is
// bound by the shared-memory histogram atomics beyond that)
constexpr int kInFlight = 4;

struct BatchPtrs {
    const void *p[kMaxBatchesPerLaunch];
};

struct CalibState {
    unsigned int max_bits;     // max |x| bit pattern (fp32 bits; bf16 widened)
    unsigned int bucket;       // fp32: pass-1 bucket holding the rank
    unsigned long long rank2;  // fp32: rank inside that bucket (1-based)
};

constexpr size_t kStateBytes = 256;

__device__ __forceinline__ uint32_t mag_bits(uint32_t raw, bool bf16)
{
    // returns the fp32 magnitude bit pattern
    return bf16 ? ((raw & 0x7FFFu) << 16) : (raw & 0x7FFFFFFFu);
}

template <bool BF16>
__global__ void __launch_bounds__(kHistThreads)
    hist1_kernel(BatchPtrs ptrs, int nb, int64_t elems, unsigned long long *__restrict__ hist,
                 CalibState *__restrict__ state)
{
    extern __shared__ uint32_t sh[]; // kBins1 counters
    for (int i = threadIdx.x; i < kBins1; i += kHistThreads)
        sh[i] = 0;
    __syncthreads();
    uint32_t mx = 0;
    constexpr int kPerVec = BF16 ? 8 : 4;
    const int64_t nvec = elems / kPerVec;
    const int64_t per_cta = (nvec + gridDim.x - 1) / gridDim.x;
    const int64_t v0 = (int64_t)blockIdx.x * per_cta;
    const int64_t v1 = min(nvec, v0 + per_cta);
    auto count = [&](const uint4 &w) {
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if constexpr (BF16) {
                const uint32_t lo = u[j] & 0x7FFFu, hi = (u[j] >> 16) & 0x7FFFu;
                atomicAdd(&sh[lo], 1u);
                atomicAdd(&sh[hi], 1u);
                mx = max(mx, max(lo, hi) << 16);
            } else {
                const uint32_t m = u[j] & 0x7FFFFFFFu;
                atomicAdd(&sh[m >> 16], 1u);
                mx = max(mx, m);
            }
        }
    };
    for (int b = 0; b < nb; ++b) {
        const uint4 *x = reinterpret_cast<const uint4 *>(ptrs.p[b]);
        // kInFlight vectors per thread per step: all loads issued before any is counted
        int64_t i = v0 + threadIdx.x;
        for (; i + (kInFlight - 1) * kHistThreads < v1; i += kInFlight * kHistThreads) {
            uint4 w[kInFlight];
#pragma unroll
            for (int k = 0; k < kInFlight; ++k)
                w[k] = __ldg(x + i + k * kHistThreads);
#pragma unroll
            for (int k = 0; k < kInFlight; ++k)
                count(w[k]);
        }
        for (; i < v1; i += kHistThreads)
            count(__ldg(x + i));
        // tail elements that do not fill a 16-byte vector: CTA 0 takes them
        if (blockIdx.x == 0) {
            for (int64_t e = nvec * kPerVec + threadIdx.x; e < elems; e += kHistThreads) {
                uint32_t m;
                if constexpr (BF16)
                    m = mag_bits(reinterpret_cast<const uint16_t *>(ptrs.p[b])[e], true);
                else
                    m = mag_bits(reinterpret_cast<const uint32_t *>(ptrs.p[b])[e], false);
                atomicAdd(&sh[m >> 16], 1u);
                mx = max(mx, m);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if ((threadIdx.x & 31) == 0)
        atomicMax(&state->max_bits, mx);
    __syncthreads();
    for (int i = threadIdx.x; i < kBins1; i += kHistThreads)
        if (sh[i])
            atomicAdd(&hist[i], (unsigned long long)sh[i]);
}

// Pass 2 (fp32): histogram of the low 16 bits of the values in the selected bucket.
__global__ void __launch_bounds__(kHistThreads)
    hist2_kernel(BatchPtrs ptrs, int nb, int64_t elems, unsigned long long *__restrict__ hist2,
                 const CalibState *__restrict__ state)
{
    const uint32_t bucket = state->bucket;
    const int64_t nvec = elems / 4;
    const int64_t stride = (int64_t)gridDim.x * kHistThreads;
    for (int b = 0; b < nb; ++b) {
        const uint4 *x = reinterpret_cast<const uint4 *>(ptrs.p[b]);
        for (int64_t i = (int64_t)blockIdx.x * kHistThreads + threadIdx.x; i < nvec;
             i += stride) {
            const uint4 w = __ldg(x + i);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t m = u[j] & 0x7FFFFFFFu;
                if ((m >> 16) == bucket)
                    atomicAdd(&hist2[m & 0xFFFFu], 1ull);
            }
        }
        if (blockIdx.x == 0)
            for (int64_t e = nvec * 4 + threadIdx.x; e < elems; e += kHistThreads) {
                const uint32_t m = reinterpret_cast<const uint32_t *>(ptrs.p[b])[e] & 0x7FFFFFFFu;
                if ((m >> 16) == bucket)
                    atomicAdd(&hist2[m & 0xFFFFu], 1ull);
            }
    }
}

// Find the bin where the running count first reaches `rank` (1-based). One CTA of 1024
// threads; each thread owns nbins/1024 consecutive bins.
__device__ void select_bin(const unsigned long long *__restrict__ hist, int nbins,
                           unsigned long long rank, int *out_bin, unsigned long long *out_before)
{
    __shared__ unsigned long long part[kHistThreads];
    const int per = nbins / kHistThreads;
    const int b0 = threadIdx.x * per;
    unsigned long long s = 0;
    for (int i = 0; i < per; ++i)
        s += hist[b0 + i];
    part[threadIdx.x] = s;
    __syncthreads();
    // inclusive scan (Hillis-Steele)
    for (int o = 1; o < kHistThreads; o <<= 1) {
        unsigned long long v = threadIdx.x >= o ? part[threadIdx.x - o] : 0ull;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    const unsigned long long incl = part[threadIdx.x];
    const unsigned long long excl = incl - s;
    if (excl < rank && rank <= incl) {
        unsigned long long c = excl;
        for (int i = 0; i < per; ++i) {
            const unsigned long long h = hist[b0 + i];
            if (c + h >= rank) {
                *out_bin = b0 + i;
                *out_before = c;
                break;
            }
            c += h;
        }
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kHistThreads)
    select1_kernel(const unsigned long long *__restrict__ hist, unsigned long long rank,
                   CalibState *__restrict__ state, float *__restrict__ out_pct,
                   float *__restrict__ out_max)
{
    __shared__ int s_bin;
    __shared__ unsigned long long s_before;
    if (threadIdx.x == 0) {
        s_bin = 0;
        s_before = 0;
    }
    __syncthreads();
    select_bin(hist, kBins1, rank, &s_bin, &s_before);
    __syncthreads();
    if (threadIdx.x == 0) {
        *out_max = __uint_as_float(state->max_bits);
        if (BF16) {
            *out_pct = __uint_as_float((uint32_t)s_bin << 16);
        } else {
            state->bucket = (unsigned int)s_bin;
            state->rank2 = rank - s_before;
        }
    }
}

__global__ void __launch_bounds__(kHistThreads)
    select2_kernel(const unsigned long long *__restrict__ hist2,
                   const CalibState *__restrict__ state, float *__restrict__ out_pct)
{
    __shared__ int s_bin;
    __shared__ unsigned long long s_before;
    if (threadIdx.x == 0) {
        s_bin = 0;
        s_before = 0;
    }
    __syncthreads();
    select_bin(hist2, kBins2, state->rank2, &s_bin, &s_before);
    __syncthreads();
    if (threadIdx.x == 0)
        *out_pct = __uint_as_float((state->bucket << 16) | (uint32_t)s_bin);
}

} // namespace

size_t calib_workspace_bytes(int is_bf16)
{
    return kStateBytes + kBins1 * 8 + (is_bf16 ? 0 : (size_t)kBins2 * 8);
}

cudaError_t launch_calib(const void *const *batches, int num_batches, int64_t elems_per_batch,
                         int is_bf16, uint64_t rank, float *out_pct, float *out_max, void *ws,
                         cudaStream_t s)
{
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    CalibState *state = reinterpret_cast<CalibState *>(w);
    unsigned long long *hist1 = reinterpret_cast<unsigned long long *>(w + kStateBytes);
    unsigned long long *hist2 = hist1 + kBins1;
    cudaError_t e = cudaMemsetAsync(ws, 0, calib_workspace_bytes(is_bf16), s);
    if (e != cudaSuccess)
        return e;
    const size_t shmem = kBins1 * sizeof(uint32_t);
    e = is_bf16 ? cudaFuncSetAttribute(hist1_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem)
                : cudaFuncSetAttribute(hist1_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem);
    if (e != cudaSuccess)
        return e;
    const int grid = num_sms();
    for (int b0 = 0; b0 < num_batches; b0 += kMaxBatchesPerLaunch) {
        BatchPtrs p{};
        const int nb = min(kMaxBatchesPerLaunch, num_batches - b0);
        for (int i = 0; i < nb; ++i)
            p.p[i] = batches[b0 + i];
        if (is_bf16)
            hist1_kernel<true><<<grid, kHistThreads, shmem, s>>>(p, nb, elems_per_batch, hist1,
                                                                 state);
        else
            hist1_kernel<false><<<grid, kHistThreads, shmem, s>>>(p, nb, elems_per_batch, hist1,
                                                                  state);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    if (is_bf16)
        select1_kernel<true><<<1, kHistThreads, 0, s>>>(hist1, rank, state, out_pct, out_max);
    else
        select1_kernel<false><<<1, kHistThreads, 0, s>>>(hist1, rank, state, out_pct, out_max);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    if (is_bf16)
        return cudaSuccess;
    for (int b0 = 0; b0 < num_batches; b0 += kMaxBatchesPerLaunch) {
        BatchPtrs p{};
        const int nb = min(kMaxBatchesPerLaunch, num_batches - b0);
        for (int i = 0; i < nb; ++i)
            p.p[i] = batches[b0 + i];
        hist2_kernel<<<grid * 4, kHistThreads, 0, s>>>(p, nb, elems_per_batch, hist2, state);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    select2_kernel<<<1, kHistThreads, 0, s>>>(hist2, state, out_pct);
    return cudaGetLastError();
}

} // namespace nvfp4
