// gemm_sm100.cu -- block-scaled W4A4 GEMM on the sm_100a FP4 tensor cores.
//
// Y = dequant(A) . dequant(W)^T with A [M x K] and W [N x K] in NVFP4: E2M1 codes, one E4M3
// scale per 16 values along K, one fp32 global scale per tensor ("Qwen-Image NVFP4 on a 16 GB
// Ada GPU", "What NVFP4 is and how it differs from NF4": on Blackwell the tensor cores
// multiply in FP4 with weights and activations both in 4 bits).
//
// Kernel structure (one CTA per SM, persistent over work units):
//   warp 0      TMA producer: per 256-wide k-tile loads the A tile (128 rows x 128 B of packed
//               codes), the B tile (BN rows x 128 B), both 128B-swizzled, and the scale-factor
//               atoms of both (512-byte atoms of the tensor-core scale layout) into a
//               STAGES-deep shared-memory ring; completion is tracked by mbarrier tx counts.
//   warp 1      MMA issuer (one thread): copies the k-tile's scale atoms shared -> TMEM with
//               tcgen05.cp (32x128b, replicated to the four lane quarters), then issues four
//               tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X (M128 x BN x K64) into a
//               fp32 accumulator in TMEM, and frees the ring slot with tcgen05.commit.
//               Also allocates / frees TMEM.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp owns one 32-lane quarter),
//               times alpha = sgA * sgW, cast, store (or raw fp32 partials for split-K).
// Small M (<= 128) runs swap-AB: the weights take the MMA's M side (128 rows of W per tile)
// and the activation rows the N side (8..128), so the tensor cores stream the weight matrix
// at full width; with few tiles the K range is split over CTAs and a second kernel adds the
// fp32 partials in split order (deterministic).
// Every wait is bounded; a wait that gives up records NVFP4_ERR_TIMEOUT in the library's
// status word, lets the CTA drain its in-flight copies / MMAs, frees TMEM and returns.
// No TMA multicast is used.
#include <cuda.h>
#include <mutex>

#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int BM = 128;
constexpr int kThreads = 192;
constexpr uint32_t kWaitLimit = 1u << 20;

template <int BN> struct Cfg {
    static constexpr int kStages = BN == 256 ? 4 : (BN == 128 ? 6 : 7);
    static constexpr int kSfbBands = BN > 128 ? 2 : 1;
    static constexpr int kABytes = BM * 128;
    static constexpr int kBBytes = BN * 128;
    static constexpr int kSfaBytes = 4 * 512;
    static constexpr int kSfbBytes = kSfbBands * 4 * 512;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kOffB = kStages * kABytes;
    static constexpr int kOffSfa = kOffB + kStages * kBBytes;
    static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
    static constexpr int kOffBar = kOffSfb + kStages * kSfbBytes;
    static constexpr int kSmemBytes = 1024 + kOffBar + 256;
    // TMEM columns: accumulator, then double-buffered scale factors.
    static constexpr int kAccCols = BN < 32 ? 32 : BN;
    static constexpr int kSfaCol = kAccCols;
    static constexpr int kSfbCol = kSfaCol + 2 * 16;
    static constexpr int kSfbColsPerKb = 4 * kSfbBands;
    static constexpr int kUsedCols = kSfbCol + 2 * 4 * kSfbColsPerKb;
    static constexpr int kTmemCols = kUsedCols <= 32    ? 32
                                     : kUsedCols <= 64  ? 64
                                     : kUsedCols <= 128 ? 128
                                     : kUsedCols <= 256 ? 256
                                                        : 512;
    static constexpr uint32_t kTx = kStageBytes;
    // instruction descriptor: E2M1 x E2M1, K-major both, UE4M3 scales, M = 128, N = BN
    static constexpr uint32_t kIdesc =
        (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kUsedCols <= 512, "TMEM budget");
};

struct GemmParams {
    int64_t rows_a, rows_b;    // valid rows of the MMA A / B operands
    int64_t tiles_a, tiles_b;  // tiles of 128 / BN rows
    int kt_total, kt_per_split, splits;
    int64_t units;             // tiles_a * tiles_b * splits
    const float *a_gs, *w_gs;  // global scales (device)
    void *y;
    int64_t ldy;               // = N
    int out_bf16, swap;
    float *partial;            // split-K partials [splits][tiles_a*128][tiles_b*BN]
    int *status;
};

__device__ __forceinline__ void set_timeout(int *status)
{
    atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
}

template <int BN>
__device__ __forceinline__ void store_chunk(const GemmParams &p, int64_t arow, int64_t bcol0,
                                            int split, const uint32_t *v, int n, float alpha)
{
    if (arow >= p.rows_a)
        return;
    if (p.splits > 1) {
        float *dst = p.partial + ((int64_t)split * p.tiles_a * BM + arow) * (p.tiles_b * BN) + bcol0;
        if (n % 4 == 0) {
            for (int j = 0; j < n; j += 4)
                *reinterpret_cast<float4 *>(dst + j) =
                    make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        } else {
            for (int j = 0; j < n; ++j)
                dst[j] = __uint_as_float(v[j]);
        }
        return;
    }
    if (p.swap) {
        // A row = output column n, B rows = output rows m
        for (int j = 0; j < n; ++j) {
            const int64_t m = bcol0 + j;
            if (m >= p.rows_b)
                break;
            const float r = __uint_as_float(v[j]) * alpha;
            if (p.out_bf16)
                reinterpret_cast<__nv_bfloat16 *>(p.y)[m * p.ldy + arow] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float *>(p.y)[m * p.ldy + arow] = r;
        }
        return;
    }
    // A row = output row m, B rows = output columns
    const int64_t base = arow * p.ldy + bcol0;
    const bool full = bcol0 + n <= p.rows_b;
    if (p.out_bf16) {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.y) + base;
        if (full && (p.ldy % 8 == 0) && (n % 8 == 0)) {
            for (int j = 0; j < n; j += 8) {
                uint32_t w[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[j + 2 * t]) * alpha,
                                                             __uint_as_float(v[j + 2 * t + 1]) * alpha);
                    w[t] = *reinterpret_cast<uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else {
            for (int j = 0; j < n && bcol0 + j < p.rows_b; ++j)
                dst[j] = __float2bfloat16_rn(__uint_as_float(v[j]) * alpha);
        }
    } else {
        float *dst = reinterpret_cast<float *>(p.y) + base;
        if (full && (p.ldy % 4 == 0) && (n % 4 == 0)) {
            for (int j = 0; j < n; j += 4)
                *reinterpret_cast<float4 *>(dst + j) =
                    make_float4(__uint_as_float(v[j]) * alpha, __uint_as_float(v[j + 1]) * alpha,
                                __uint_as_float(v[j + 2]) * alpha,
                                __uint_as_float(v[j + 3]) * alpha);
        } else {
            for (int j = 0; j < n && bcol0 + j < p.rows_b; ++j)
                dst[j] = __uint_as_float(v[j]) * alpha;
        }
    }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSFA,
                      const __grid_constant__ CUtensorMap tmSFB, const GemmParams p)
{
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *acc_full = empty_bar + C::kStages;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain_bar = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 3);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drain_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles_ab = p.tiles_a * p.tiles_b;

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmSFA);
            tma_prefetch_desc(&tmSFB);
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
                const int split = (int)(u / tiles_ab);
                const int64_t rem = u - (int64_t)split * tiles_ab;
                const int64_t ta = rem % p.tiles_a, tb = rem / p.tiles_a;
                const int k0 = split * p.kt_per_split;
                const int k1 = min(p.kt_total, k0 + p.kt_per_split);
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kWaitLimit)) {
                        set_timeout(p.status);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kABytes;
                    uint8_t *sb = smem + C::kOffB + stage * C::kBBytes;
                    uint8_t *ssfa = smem + C::kOffSfa + stage * C::kSfaBytes;
                    uint8_t *ssfb = smem + C::kOffSfb + stage * C::kSfbBytes;
                    mbar_arrive_expect_tx(&full_bar[stage], C::kTx);
                    tma_load_2d(sa, &tmA, &full_bar[stage], kt * 128, (int)(ta * BM));
                    tma_load_2d(sb, &tmB, &full_bar[stage], kt * 128, (int)(tb * BN));
                    tma_load_3d(ssfa, &tmSFA, &full_bar[stage], 0, kt * 4, (int)ta);
                    tma_load_3d(ssfb, &tmSFB, &full_bar[stage], 0, kt * 4,
                                (int)((tb * BN) >> 7));
                    ++issued;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Drain: make sure every copy this thread issued has landed before exit.
            int s = stage;
            uint32_t ph = phase;
            const int64_t last = issued < C::kStages ? issued : C::kStages;
            for (int64_t i = 0; i < last; ++i) {
                if (--s < 0) {
                    s = C::kStages - 1;
                    ph ^= 1;
                }
                if (!mbar_wait(&full_bar[s], ph, kWaitLimit))
                    set_timeout(p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0, sfbuf = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
            const int split = (int)(u / tiles_ab);
            const int k0 = split * p.kt_per_split;
            const int k1 = min(p.kt_total, k0 + p.kt_per_split);
            if (!mbar_wait(acc_empty, acc_phase ^ 1, kWaitLimit)) {
                if (lane == 0)
                    set_timeout(p.status);
                break;
            }
            tc_fence_after();
            for (int kt = k0; kt < k1; ++kt) {
                if (!mbar_wait(&full_bar[stage], phase, kWaitLimit)) {
                    if (lane == 0)
                        set_timeout(p.status);
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t ssfa = smem_u32(smem + C::kOffSfa + stage * C::kSfaBytes);
                    const uint32_t ssfb = smem_u32(smem + C::kOffSfb + stage * C::kSfbBytes);
                    const uint32_t tsfa = tmem + C::kSfaCol + sfbuf * 16;
                    const uint32_t tsfb = tmem + C::kSfbCol + sfbuf * (4 * C::kSfbColsPerKb);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        tc_cp_sf_atom(tsfa + kb * 4,
                                      smem_desc(ssfa + kb * 512, 0, 128, kLayoutSwizzleNone));
#pragma unroll
                        for (int h = 0; h < C::kSfbBands; ++h)
                            tc_cp_sf_atom(tsfb + kb * C::kSfbColsPerKb + h * 4,
                                          smem_desc(ssfb + (h * 4 + kb) * 512, 0, 128,
                                                    kLayoutSwizzleNone));
                    }
                    const uint64_t adesc = smem_desc(smem_u32(smem + stage * C::kABytes), 16,
                                                     1024, kLayoutSwizzle128B);
                    const uint64_t bdesc =
                        smem_desc(smem_u32(smem + C::kOffB + stage * C::kBBytes), 16, 1024,
                                  kLayoutSwizzle128B);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        // advance 32 bytes (64 FP4 values) along K inside the swizzle atom
                        tc_mma_nvf4(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb),
                                    C::kIdesc, tsfa + kb * 4, tsfb + kb * C::kSfbColsPerKb,
                                    (kt > k0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty_bar[stage]);
                }
                __syncwarp();
                sfbuf ^= 1;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok)
                break;
            if (lane == 0)
                tc_commit(acc_full);
            __syncwarp();
            acc_phase ^= 1;
        }
        // Drain: every MMA / copy issued by this thread completes before TMEM is freed.
        if (lane == 0) {
            tc_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0, kWaitLimit))
                set_timeout(p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue -----------------------------------
        const int q = warp & 3; // TMEM lane quarter this warp may access
        const float alpha = __fmul_rn(*p.a_gs, *p.w_gs);
        uint32_t acc_phase = 0;
        for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x) {
            const int split = (int)(u / tiles_ab);
            const int64_t rem = u - (int64_t)split * tiles_ab;
            const int64_t ta = rem % p.tiles_a, tb = rem / p.tiles_a;
            if (!mbar_wait(acc_full, acc_phase, kWaitLimit)) {
                if (lane == 0)
                    set_timeout(p.status);
                break;
            }
            tc_fence_after();
            const int64_t arow = ta * BM + q * 32 + lane;
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
            if constexpr (BN >= 32) {
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(trow + c0, v);
                    tmem_ld_wait();
                    store_chunk<BN>(p, arow, tb * BN + c0, split, v, 32, alpha);
                }
            } else if constexpr (BN == 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(trow, v);
                tmem_ld_wait();
                store_chunk<BN>(p, arow, tb * BN, split, v, 16, alpha);
            } else {
                uint32_t v[8];
                tmem_ld_32x32b_x8(trow, v);
                tmem_ld_wait();
                store_chunk<BN>(p, arow, tb * BN, split, v, 8, alpha);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acc_empty);
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Sum split-K partials in split order, scale by alpha, cast, store.
__global__ void splitk_reduce_kernel(const float *__restrict__ partial, int splits,
                                     int64_t rows_a, int64_t rows_b, int64_t a_pad,
                                     int64_t b_pad, const float *__restrict__ a_gs,
                                     const float *__restrict__ w_gs, void *__restrict__ y,
                                     int64_t ldy, int out_bf16, int swap)
{
    const float alpha = __fmul_rn(*a_gs, *w_gs);
    const int64_t total = rows_a * rows_b;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t a, b;
        if (swap) {
            a = i % rows_a;
            b = i / rows_a;
        } else {
            a = i / rows_b;
            b = i % rows_b;
        }
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s)
            acc += partial[((int64_t)s * a_pad + a) * b_pad + b];
        const float r = acc * alpha;
        const int64_t off = swap ? (b * ldy + a) : (a * ldy + b);
        if (out_bf16)
            reinterpret_cast<__nv_bfloat16 *>(y)[off] = __float2bfloat16_rn(r);
        else
            reinterpret_cast<float *>(y)[off] = r;
    }
}

// ---------------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// Packed codes [rows x K/2] bytes, box 128 B x box_rows, 128B swizzle.
bool make_codes_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K, int box_rows)
{
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Swizzled scales viewed as [bands][atoms][128 x u32]; box = 4 atoms x box_bands bands.
bool make_sf_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K, int box_bands)
{
    const int64_t apb = (K / 16 + 3) / 4;
    const int64_t bands = (rows + 127) / 128;
    cuuint64_t dims[3] = {128u, (cuuint64_t)apb, (cuuint64_t)bands};
    cuuint64_t strides[2] = {512u, (cuuint64_t)(apb * 512)};
    cuuint32_t box[3] = {128u, 4u, (cuuint32_t)box_bands};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_bn(const LinearPlan &pl, const uint8_t *a_codes, const uint8_t *a_sf,
                      const uint8_t *b_codes, const uint8_t *b_sf, int64_t K, GemmParams gp,
                      cudaStream_t s, nvfp4_status *st)
{
    using C = Cfg<BN>;
    CUtensorMap tmA, tmB, tmSFA, tmSFB;
    if (!encode_fn() || !make_codes_map(&tmA, a_codes, pl.rows_a, K, BM) ||
        !make_codes_map(&tmB, b_codes, pl.rows_b, K, BN) ||
        !make_sf_map(&tmSFA, a_sf, pl.rows_a, K, 1) ||
        !make_sf_map(&tmSFB, b_sf, pl.rows_b, K, C::kSfbBands)) {
        *st = NVFP4_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    static std::once_flag flags[64];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t attr_err = cudaSuccess;
    std::call_once(flags[dev & 63], [&]() {
        attr_err = cudaFuncSetAttribute(nvfp4_gemm_kernel<BN>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return attr_err;
    int64_t grid = gp.units < num_sms() ? gp.units : num_sms();
    if (grid < 1)
        grid = 1;
    nvfp4_gemm_kernel<BN><<<(unsigned)grid, kThreads, C::kSmemBytes, s>>>(tmA, tmB, tmSFA,
                                                                          tmSFB, gp);
    return cudaGetLastError();
}

} // namespace

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K)
{
    LinearPlan p{};
    p.kt = (int)((K + 255) / 256);
    if (M <= 128) {
        p.swap_ab = true;
        p.bn = M <= 8 ? 8 : M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
        p.rows_a = N;
        p.rows_b = M;
    } else {
        p.swap_ab = false;
        p.bn = 256;
        p.rows_a = M;
        p.rows_b = N;
    }
    p.tiles_a = (p.rows_a + 127) / 128;
    p.tiles_b = (p.rows_b + p.bn - 1) / p.bn;
    p.splits = 1;
    p.kt_per_split = p.kt;
    const int64_t tiles = p.tiles_a * p.tiles_b;
    const int sms = num_sms();
    if (tiles > 0 && p.kt > 1 && tiles * 2 <= sms) {
        int64_t sp = sms / tiles;
        if (sp > p.kt)
            sp = p.kt;
        p.kt_per_split = (int)((p.kt + sp - 1) / sp);
        p.splits = (p.kt + p.kt_per_split - 1) / p.kt_per_split;
    }
    p.ws_bytes = p.splits > 1
                     ? (size_t)p.splits * p.tiles_a * 128 * p.tiles_b * p.bn * sizeof(float)
                     : 0;
    return p;
}

cudaError_t launch_linear(const LinearPlan &pl, const uint8_t *a_codes, const uint8_t *a_sf,
                          const float *a_gs, const uint8_t *w_codes, const uint8_t *w_sf,
                          const float *w_gs, int64_t M, int64_t N, int64_t K, int out_bf16,
                          void *y, void *ws, cudaStream_t s, nvfp4_status *st)
{
    GemmParams gp{};
    gp.rows_a = pl.rows_a;
    gp.rows_b = pl.rows_b;
    gp.tiles_a = pl.tiles_a;
    gp.tiles_b = pl.tiles_b;
    gp.kt_total = pl.kt;
    gp.kt_per_split = pl.kt_per_split;
    gp.splits = pl.splits;
    gp.units = pl.tiles_a * pl.tiles_b * pl.splits;
    gp.a_gs = a_gs;
    gp.w_gs = w_gs;
    gp.y = y;
    gp.ldy = N;
    gp.out_bf16 = out_bf16;
    gp.swap = pl.swap_ab ? 1 : 0;
    gp.partial = reinterpret_cast<float *>(ws);
    gp.status = device_status_ptr();
    // MMA operand A is the 128-row side; B the BN-row side.
    const uint8_t *ca = pl.swap_ab ? w_codes : a_codes;
    const uint8_t *sa = pl.swap_ab ? w_sf : a_sf;
    const uint8_t *cb = pl.swap_ab ? a_codes : w_codes;
    const uint8_t *sb = pl.swap_ab ? a_sf : w_sf;
    cudaError_t e;
    switch (pl.bn) {
    case 8: e = launch_bn<8>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    case 16: e = launch_bn<16>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    case 32: e = launch_bn<32>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    case 64: e = launch_bn<64>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    case 128: e = launch_bn<128>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    default: e = launch_bn<256>(pl, ca, sa, cb, sb, K, gp, s, st); break;
    }
    if (e != cudaSuccess || pl.splits == 1)
        return e;
    const int64_t total = pl.rows_a * pl.rows_b;
    int64_t g = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap)
        g = cap;
    splitk_reduce_kernel<<<(unsigned)g, 256, 0, s>>>(
        reinterpret_cast<const float *>(ws), pl.splits, pl.rows_a, pl.rows_b, pl.tiles_a * 128,
        pl.tiles_b * pl.bn, a_gs, w_gs, y, N, out_bf16, pl.swap_ab ? 1 : 0);
    return cudaGetLastError();
}

} // namespace nvfp4
