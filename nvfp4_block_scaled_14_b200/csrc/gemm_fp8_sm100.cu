// gemm_fp8_sm100.cu -- FP8 E4M3 tensorwise W8A8 linear layer on the sm_100a tensor cores.
//
// Y = (sA * sW) * A8 . W8^T with A8 [M x K] and W8 [N x K] E4M3 codes and one fp32 scale per
// tensor ("Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details" and "Layer breakdown":
// embed_tokens and lm_head in float8_e4m3fn, tensorwise; "Runtime / hardware": FP8 layers run
// as native FP8 on Blackwell. "Qwen-Rapid-AIO FP8 -> NVFP4", "Solution": layers that are FP8
// stay FP8, so weights that arrive as E4M3 with their scale are used as they are).
//
// CTA pairs (clusters of 2) compute 256 x 256 output tiles, persistent over the tiles, with
// tcgen05.mma.cta_group::2.kind::f8f6f4 (M256 N256 K32, E4M3 x E4M3, fp32 accumulation in
// TMEM) issued by the leader CTA. Each CTA loads its 128 rows of A and its 128 rows of W per
// 128-value k-tile (TMA, 128B swizzle, no multicast) into a 5-stage ring. With no block scales
// TMEM holds two 256-column accumulators, so a finished tile is read out while the next one
// accumulates.
//   warp 0     TMA producer (both CTAs; the loads signal the leader's barrier)
//   warp 1     MMA issuer (leader) -- also allocates / frees TMEM
//   warps 2..5 epilogue (both CTAs): TMEM -> x alpha -> bf16 -> shared staging -> TMA store;
//              fp32 output or a row stride the TMA store cannot take: direct stores
// Every wait is bounded; a wait that gives up records NVFP4_ERR_TIMEOUT and the CTA drains.
#include <cuda.h>
#include <cstring>
#include <mutex>

#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kF8Threads = 192;
constexpr uint32_t kF8WaitLimit = 1u << 20;

struct F8 {
    static constexpr int kStages = 5;
    static constexpr int kABytes = 128 * 128; // 128 rows x 128 bytes (128 E4M3 values of K)
    static constexpr int kBBytes = 128 * 128;
    static constexpr int kOffB = kStages * kABytes;
    static constexpr int kOffStaging = kOffB + kStages * kBBytes;
    static constexpr int kStagingBytes = 128 * 256 * 2; // one CTA's 128 x 256 bf16 rows
    static constexpr int kOffBar = kOffStaging + kStagingBytes;
    static constexpr int kSmemBytes = kOffBar + 256;
    static constexpr uint32_t kTx = 2 * (kABytes + kBBytes); // both CTAs, on the leader
    static constexpr int kTmemCols = 512;                    // two 256-column accumulators
    // instruction descriptor of kind::f8f6f4: D fp32 (bits 4-5 = 1), A and B E4M3 (format 0),
    // both K-major, N >> 3 at bit 17, M >> 4 at bit 24
    static constexpr uint32_t kIdesc =
        (1u << 4) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct F8Params {
    int64_t M, N;
    int64_t tiles_a, tiles_b; // 256-row / 256-column tiles
    int kt_total;             // 128-value k-tiles
    const float *a_scale, *w_scale;
    void *y;
    int out_bf16;
    int tma_store;
    int *status;
};

__device__ __forceinline__ void f8_set_timeout(int *status)
{
    atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
}

__device__ __forceinline__ void tc_mma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

__device__ __forceinline__ uint32_t f8_pack_bf16x2(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// This thread's 256-column accumulator row x alpha -> bf16 into row r of the staging tile:
// four 128-row x 128-byte boxes, 16-byte chunks swizzled by row % 8 (the TMA store's 128B
// swizzle). Four TMEM loads in flight per wait.
__device__ __forceinline__ void f8_stage_row(uint32_t trow, uint32_t stg, int r, float alpha)
{
#pragma unroll 1
    for (int c0 = 0; c0 < 256; c0 += 64) {
        uint32_t v[64];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tmem_ld_32x32b_x16(trow + c0 + 16 * i, v + 16 * i);
        tmem_ld_wait();
        const uint32_t box = stg + (c0 >> 6) * (128 * 128) + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = f8_pack_bf16x2(__uint_as_float(v[8 * ch + 2 * j]) * alpha,
                                      __uint_as_float(v[8 * ch + 2 * j + 1]) * alpha);
            sts128(box + ((ch ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
    }
}

// Direct stores of this thread's row (fp32 output, or bf16 with a row stride the TMA store
// cannot take), 32 columns per TMEM wait, bounds-checked.
__device__ __forceinline__ void f8_store_row(const F8Params &p, uint32_t trow, int64_t row,
                                             int64_t col0, float alpha)
{
#pragma unroll 1
    for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x16(trow + c0, v);
        tmem_ld_32x32b_x16(trow + c0 + 16, v + 16);
        tmem_ld_wait();
        if (row >= p.M)
            continue;
        const int64_t base = row * p.N + col0 + c0;
        if (p.out_bf16) {
            __nv_bfloat16 *y = reinterpret_cast<__nv_bfloat16 *>(p.y) + base;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (col0 + c0 + j < p.N)
                    y[j] = __float2bfloat16_rn(__uint_as_float(v[j]) * alpha);
        } else {
            float *y = reinterpret_cast<float *>(p.y) + base;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (col0 + c0 + j < p.N)
                    y[j] = __uint_as_float(v[j]) * alpha;
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kF8Threads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmY, const F8Params p)
{
    using C = F8;
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0)
            atomicExch(p.status, (int)NVFP4_ERR_CUDA);
        return; // uniform across the cluster: both CTAs see the same layout
    }
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kOffBar); // leader only
    uint64_t *empty_bar = full_bar + C::kStages;                         // both
    uint64_t *acc_full = empty_bar + C::kStages;                         // both, [2]
    uint64_t *acc_empty = acc_full + 2;                                  // leader only, [2]
    uint64_t *drain_bar = acc_empty + 2;                                 // leader only
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8); // four epilogue warps in each CTA
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync(); // barriers of both CTAs initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles = p.tiles_a * p.tiles_b;
    const int64_t cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (warp == 0) {
        // ------------------------------- TMA producer (both CTAs) ---------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            pdl_wait(); // operands come from the stream's earlier kernels
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t u = cluster_id; u < tiles && ok; u += nclusters) {
                const int64_t ta = u % p.tiles_a, tb = u / p.tiles_a;
                const int arow = (int)(ta * 256 + rank * 128);
                const int brow = (int)(tb * 256 + rank * 128);
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kF8WaitLimit)) {
                        f8_set_timeout(p.status);
                        ok = false;
                        break;
                    }
                    const uint32_t leader_full = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (leader)
                        mbar_arrive_expect_tx(&full_bar[stage], C::kTx);
                    tma_load_2d_pair(smem + stage * C::kABytes, &tmA, leader_full, kt * 128, arow);
                    tma_load_2d_pair(smem + C::kOffB + stage * C::kBBytes, &tmB, leader_full,
                                     kt * 128, brow);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer (leader) ---------------------------
        if (leader) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phases = 0u; // bit b: phase of accumulator b
            int buf = 0;
            bool ok = true;
            for (int64_t u = cluster_id; u < tiles && ok; u += nclusters) {
                if (!mbar_wait(&acc_empty[buf], ((acc_phases >> buf) & 1u) ^ 1u, kF8WaitLimit)) {
                    if (lane == 0)
                        f8_set_timeout(p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t tacc = tmem + (uint32_t)(buf * 256);
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait(&full_bar[stage], phase, kF8WaitLimit)) {
                        if (lane == 0)
                            f8_set_timeout(p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint64_t adesc = smem_desc(smem_u32(smem + stage * C::kABytes), 16,
                                                         1024, kLayoutSwizzle128B);
                        const uint64_t bdesc =
                            smem_desc(smem_u32(smem + C::kOffB + stage * C::kBBytes), 16, 1024,
                                      kLayoutSwizzle128B);
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) // K32 = 32 bytes per MMA
                            tc_mma_f8_pair(tacc, adesc + (uint64_t)(2 * kb),
                                           bdesc + (uint64_t)(2 * kb), C::kIdesc,
                                           (kt > 0 || kb > 0) ? 1u : 0u);
                        tc_commit_pair_mc(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok)
                    break;
                if (lane == 0)
                    tc_commit_pair_mc(&acc_full[buf], 0x3);
                __syncwarp();
                acc_phases ^= 1u << buf;
                buf ^= 1;
            }
            if (lane == 0) {
                tc_commit_pair(drain_bar);
                if (!mbar_wait(drain_bar, 0, kF8WaitLimit))
                    f8_set_timeout(p.status);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------- epilogue (both CTAs, warps 2..5) -------------
        const int q = warp & 3;
        pdl_wait(); // tensor scales (and Y's previous readers) belong to earlier kernels
        const float alpha = __fmul_rn(*p.a_scale, *p.w_scale);
        uint32_t acc_phases = 0u;
        int buf = 0;
        for (int64_t u = cluster_id; u < tiles; u += nclusters) {
            const int64_t ta = u % p.tiles_a, tb = u / p.tiles_a;
            if (!mbar_wait(&acc_full[buf], (acc_phases >> buf) & 1u, kF8WaitLimit)) {
                if (lane == 0)
                    f8_set_timeout(p.status);
                break;
            }
            tc_fence_after();
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 256);
            const int64_t yrow = ta * 256 + rank * 128;
            if (p.tma_store) {
                if (threadIdx.x == 64)
                    bulk_wait_group_read0(); // the previous tile's stores have read the staging
                named_bar_sync(1, 128);
                f8_stage_row(trow, smem_u32(smem + C::kOffStaging), q * 32 + lane, alpha);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_remote(mapa_shared(smem_u32(&acc_empty[buf]), 0));
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (threadIdx.x == 64) {
                    // boxes that start past the last row or column of Y hold nothing to store
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (yrow < p.M && tb * 256 + b * 64 < p.N)
                            tma_store_2d(&tmY, smem + C::kOffStaging + b * (128 * 128),
                                         (int)(tb * 256 + b * 64), (int)yrow);
                    bulk_commit_group();
                }
            } else {
                f8_store_row(p, trow, yrow + q * 32 + lane, tb * 256, alpha);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_remote(mapa_shared(smem_u32(&acc_empty[buf]), 0));
            }
            acc_phases ^= 1u << buf;
            buf ^= 1;
        }
    }

    pdl_launch_dependents(); // all of this CTA's work is issued: the next kernel may launch
    if (threadIdx.x == 64)
        bulk_wait_group0();
    tc_fence_before();
    cluster_sync(); // no CTA leaves while its pair may still signal its barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------

typedef CUresult (*F8EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

F8EncodeTiledFn f8_encode_fn()
{
    static F8EncodeTiledFn fn = []() -> F8EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<F8EncodeTiledFn>(ptr);
    }();
    return fn;
}

// E4M3 codes [rows x K] bytes, box 128 bytes x 128 rows, 128B swizzle (zero fill past the edges).
bool f8_operand_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K)
{
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    return f8_encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 Y [rows x cols], box 64 columns x 128 rows, 128B swizzle (TMA store).
bool f8_out_map(CUtensorMap *m, void *base, int64_t rows, int64_t cols)
{
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {64u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    return f8_encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace

cudaError_t launch_linear_e4m3(const uint8_t *a, const float *a_scale, const uint8_t *w,
                               const float *w_scale, int64_t M, int64_t N, int64_t K, int out_bf16,
                               void *y, cudaStream_t s)
{
    if (M <= 0 || N <= 0)
        return cudaSuccess;
    F8Params p{};
    p.M = M;
    p.N = N;
    p.tiles_a = (M + 255) / 256;
    p.tiles_b = (N + 255) / 256;
    p.kt_total = (int)((K + 127) / 128);
    p.a_scale = a_scale;
    p.w_scale = w_scale;
    p.y = y;
    p.out_bf16 = out_bf16;
    p.tma_store = (out_bf16 && N % 8 == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0) ? 1 : 0;
    p.status = device_status_ptr();
    CUtensorMap tmA, tmB, tmY;
    std::memset(&tmY, 0, sizeof(tmY));
    if (!f8_encode_fn() || !f8_operand_map(&tmA, a, M, K) || !f8_operand_map(&tmB, w, N, K) ||
        (p.tma_store && !f8_out_map(&tmY, y, M, N)))
        return cudaErrorInvalidValue;
    static std::once_flag flags[64];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t attr_err = cudaSuccess;
    std::call_once(flags[dev & 63], [&]() {
        attr_err = cudaFuncSetAttribute(fp8_gemm_pair_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, F8::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return attr_err;
    const int64_t tiles = p.tiles_a * p.tiles_b;
    int64_t clusters = num_sms() / 2;
    if (clusters > tiles)
        clusters = tiles;
    if (clusters < 1)
        clusters = 1;
    // programmatic dependent launch: set-up overlaps the previous kernel's tail; the producer
    // and the epilogue wait for it before touching its outputs
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    cfg.blockDim = dim3(kF8Threads, 1, 1);
    cfg.dynamicSmemBytes = F8::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fp8_gemm_pair_kernel, tmA, tmB, tmY, p);
}

} // namespace nvfp4
