// gemm_sm100.cu -- block-scaled W4A4 GEMM on the sm_100a FP4 tensor cores.
//
// Y = dequant(A) . dequant(W)^T with A [M x K] and W [N x K] in NVFP4: E2M1 codes, one E4M3
// scale per 16 values along K, one fp32 global scale per tensor ("Qwen-Image NVFP4 on a 16 GB
// Ada GPU", "What NVFP4 is and how it differs from NF4": on Blackwell the tensor cores
// multiply in FP4 with weights and activations both in 4 bits).
//
// Kernel structure (one CTA per SM, persistent over work units, 10 warps):
//   warp 0      TMA producer: per 256-wide k-tile loads the A tile (128 rows x 128 B of packed
//               codes), the B tile (BN rows x 128 B), both 128B-swizzled, and the scale-factor
//               atoms of both (512-byte atoms of the tensor-core scale layout) into a
//               STAGES-deep shared-memory ring; completion is tracked by mbarrier tx counts.
//   warps 6..9  scale-factor feeders: move each k-tile's scale atoms shared -> registers ->
//               TMEM with tcgen05.st (every lane quarter receives the full atom, the layout
//               the block-scaled MMA reads), into one of kSfSlots TMEM slots. Doing this on
//               the SIMT side keeps it off the tensor pipe, where a tcgen05.cp per atom would
//               serialize with the MMAs.
//   warp 1      MMA issuer (one thread): per k-tile four
//               tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X (M128 x BN x K64) into a
//               fp32 accumulator in TMEM; tcgen05.commit frees the smem stage and the SF slot.
//               Also allocates / frees TMEM.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp owns one 32-lane quarter),
//               times alpha = sgA * sgW, cast to bf16 and held in registers; the accumulator
//               is released to the MMA warp before the global stores, so the stores overlap
//               the next tile's mainloop. (fp32 outputs / split-K partials store chunk-wise.)
// Large M with few tiles splits K over CTAs of this kernel and a second kernel adds the fp32
// partials in split order (deterministic).
// Large M with bf16 output (and the NVFP4-output epilogue and the low-rank branch) runs
// nvfp4_gemm_pair_kernel instead: the two CTAs of a cluster share 256 x 256 tiles
// (tcgen05 cta_group::2, M256 x N256 x K64 MMAs issued by the leader; each CTA loads 128 rows
// of A and 128 rows of B and holds its 128 rows of the accumulator), with the same warp roles.
// Its bf16 epilogue stores the first half of a tile before it hands the accumulator back and
// the second half after; the NVFP4-output form parks half of the accumulator in spare TMEM
// columns and the other half in shared memory, so the whole tile is activated and quantized
// while the next tile's MMAs run.
// Small M (<= 128) runs swap-AB in its own kernel (nvfp4_gemm_smallm_kernel): the weights take
// the MMA's M side (128 rows of W per tile) and the activation rows the N side (8..128), so
// the tensor cores stream the weight matrix at full width; K is split over a thread-block
// cluster and the partials are summed through distributed shared memory.
// Every wait is bounded; a wait that gives up records NVFP4_ERR_TIMEOUT in the library's
// status word, lets the CTA drain its in-flight copies / MMAs, frees TMEM and returns.
// No TMA multicast is used.
#include <cuda.h>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "nvfp4_encode.cuh"
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int BM = 128;
constexpr int kThreads = 320;
constexpr uint32_t kWaitLimit = 1u << 20;
#ifndef NVFP4_STAGES_256
#define NVFP4_STAGES_256 3
#endif
#ifndef NVFP4_PAIR_KERNEL
#define NVFP4_PAIR_KERNEL 1
#endif
constexpr bool kUsePairKernel = NVFP4_PAIR_KERNEL != 0;

// Shared-memory / TMEM layout of the 1-SM kernels for a B tile of BN rows and STAGES stages.
template <int BN, int STAGES = (BN == 256 ? NVFP4_STAGES_256 : (BN == 128 ? 6 : 7))> struct Cfg {
    static constexpr int kStages = STAGES;
    static constexpr int kSfbBands = BN > 128 ? 2 : 1;
    static constexpr int kABytes = BM * 128;
    static constexpr int kBBytes = BN * 128;
    static constexpr int kSfaBytes = 4 * 512;
    static constexpr int kSfbBytes = kSfbBands * 4 * 512;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kOffB = kStages * kABytes;
    static constexpr int kOffSfa = kOffB + kStages * kBBytes;
    static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
    // bf16 output staging for the TMA-store epilogue (BN = 256): four 128-row x 128-byte
    // boxes, 128B-swizzled
    static constexpr int kStagingBytes = BN == 256 ? BM * BN * 2 : 0;
    static constexpr int kOffStaging = kOffSfb + kStages * kSfbBytes;
    static constexpr int kOffBar = kOffStaging + kStagingBytes;
    static constexpr int kSmemBytes = kOffBar + 512;
    // TMEM columns: accumulator, then kSfSlots scale-factor slots; a slot holds one k-tile:
    // SFA in 16 columns (4 k-blocks x 4), SFB in 4 * kSfbColsPerKb columns.
    static constexpr int kAccCols = BN < 32 ? 32 : BN;
    static constexpr int kSfSlots = 4;
    static constexpr int kSfbColsPerKb = 4 * kSfbBands;
    static constexpr int kSlotCols = 16 + 4 * kSfbColsPerKb;
    static constexpr int kSfCol = kAccCols;
    static constexpr int kUsedCols = kSfCol + kSfSlots * kSlotCols;
    static constexpr int kTmemCols = kUsedCols <= 32    ? 32
                                     : kUsedCols <= 64  ? 64
                                     : kUsedCols <= 128 ? 128
                                     : kUsedCols <= 256 ? 256
                                                        : 512;
    static constexpr uint32_t kTx = kStageBytes;
    // instruction descriptor: E2M1 x E2M1, K-major both, UE4M3 scales, M = 128, N = BN
    static constexpr uint32_t kIdesc =
        (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static constexpr bool kResidentB = false;
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
    int tma_store; // 1: bf16 output through the shared-memory staging + TMA store
    // NVFP4 output of the pair kernel's quantizing epilogue (nvfp4_linear_nvfp4_out): codes
    // [rows_a x rows_b / 2], swizzled scales (q_apb atoms per 128-row band, q_rows_pad rows),
    // global scale from the static amax, activation (0 identity, 1 tanh-form GELU)
    uint8_t *q_codes, *q_sf;
    float *q_gs;
    const float *q_amax;
    int act, q_apb;
    int64_t q_rows_pad;
    // low-rank branch of the pair kernel (nvfp4_linear_lowrank): 64-wide k-tiles of bf16
    // T' [rows_a x r] and U [rows_b x r] after the FP4 k-tiles of each tile (0 = none)
    int lr_kt;
};

__device__ __forceinline__ void set_timeout(int *status)
{
    atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Chunk-wise store of 32 (or fewer) accumulator columns: fp32 outputs and split-K partials.
template <int BN>
__device__ __forceinline__ void store_chunk(const GemmParams &p, int64_t arow, int64_t bcol0,
                                            int split, const uint32_t *v, int n, float alpha)
{
    if (arow >= p.rows_a)
        return;
    if (p.splits > 1) {
        float *dst =
            p.partial + ((int64_t)split * p.tiles_a * BM + arow) * (p.tiles_b * BN) + bcol0;
        for (int j = 0; j < n; j += 4)
            *reinterpret_cast<float4 *>(dst + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
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
    const int64_t base = arow * p.ldy + bcol0;
    const bool full = bcol0 + n <= p.rows_b;
    if (p.out_bf16) {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.y) + base;
        for (int j = 0; j < n && bcol0 + j < p.rows_b; ++j)
            dst[j] = __float2bfloat16_rn(__uint_as_float(v[j]) * alpha);
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

// Read NC (<= 32) accumulator columns starting at `col` of this warp's lanes into v.
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t *v)
{
    if constexpr (NC == 32) {
        tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
    } else if constexpr (NC == 16) {
        tmem_ld_32x32b_x16(taddr, v);
    } else {
        tmem_ld_32x32b_x8(taddr, v);
    }
}

// 64 accumulator columns (registers v) x alpha -> bf16 into box `box` of the shared staging
// tile: four 128-row x 128-byte boxes, 16-byte chunks swizzled by row % 8 (the TMA store's 128B
// swizzle).
__device__ __forceinline__ void stage_box_bf16(const uint32_t (&v)[64], uint32_t stg, int box,
                                               int r, float alpha)
{
    const uint32_t base = stg + box * (128 * 128) + r * 128;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = pack_bf16x2(__uint_as_float(v[8 * ch + 2 * j]) * alpha,
                               __uint_as_float(v[8 * ch + 2 * j + 1]) * alpha);
        sts128(base + ((ch ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void tmem_ld_64cols(uint32_t taddr, uint32_t (&v)[64])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
        tmem_ld_32x32b_x16(taddr + 16 * i, v + 16 * i);
}

// This thread's accumulator row (256 fp32 columns of its TMEM lane) x alpha -> bf16 into the
// shared staging tile, 64 columns at a time with the next 64 columns' TMEM loads in flight while
// the current ones are converted and stored. `release` runs once every TMEM load of the row has
// completed, before the last 64 columns are converted: the MMA warp may then start the next
// tile while this thread finishes staging.
template <typename Release>
__device__ __forceinline__ void stage_tile_bf16(uint32_t trow, uint32_t stg, int r, float alpha,
                                                Release release)
{
    uint32_t va[64], vb[64];
    tmem_ld_64cols(trow, va);
    tmem_ld_wait();
    tmem_ld_64cols(trow + 64, vb);
    stage_box_bf16(va, stg, 0, r, alpha);
    tmem_ld_wait();
    tmem_ld_64cols(trow + 128, va);
    stage_box_bf16(vb, stg, 1, r, alpha);
    tmem_ld_wait();
    tmem_ld_64cols(trow + 192, vb);
    stage_box_bf16(va, stg, 2, r, alpha);
    tmem_ld_wait();
    release();
    stage_box_bf16(vb, stg, 3, r, alpha);
}

// Whole accumulator row of this thread -> bf16 pairs in registers (alpha applied).
template <int BN>
__device__ __forceinline__ void acc_row_to_bf16(uint32_t trow, float alpha, uint32_t *pk)
{
    constexpr int NC = BN < 16 ? BN : 16;
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += NC) {
        uint32_t v[NC];
        tmem_ld_cols<NC>(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < NC; j += 2)
            pk[(c0 + j) / 2] =
                pack_bf16x2(__uint_as_float(v[j]) * alpha, __uint_as_float(v[j + 1]) * alpha);
    }
}

__device__ __forceinline__ __nv_bfloat16 bf16_half(uint32_t w, int hi)
{
    __nv_bfloat16_raw r;
    r.x = (unsigned short)(hi ? (w >> 16) : (w & 0xFFFFu));
    return __nv_bfloat16(r);
}

// Y[arow, bcol0 .. bcol0+BN) from a register-held row (A rows are output rows).
template <int BN>
__device__ __forceinline__ void store_row_bf16(const GemmParams &p, int64_t arow, int64_t bcol0,
                                               const uint32_t *pk)
{
    if (arow >= p.rows_a)
        return;
    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.y) + arow * p.ldy + bcol0;
    if (bcol0 + BN <= p.rows_b && (p.ldy % 8) == 0) {
#pragma unroll
        for (int j = 0; j < BN; j += 8)
            *reinterpret_cast<uint4 *>(dst + j) =
                make_uint4(pk[j / 2], pk[j / 2 + 1], pk[j / 2 + 2], pk[j / 2 + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < BN; j += 2) {
            if (bcol0 + j < p.rows_b)
                dst[j] = bf16_half(pk[j / 2], 0);
            if (bcol0 + j + 1 < p.rows_b)
                dst[j + 1] = bf16_half(pk[j / 2], 1);
        }
    }
}

// Swap-AB: A rows are output columns, B rows (accumulator columns) are output rows; each
// store instruction of the warp covers 32 consecutive output columns.
template <int BN>
__device__ __forceinline__ void store_row_bf16_swap(const GemmParams &p, int64_t arow,
                                                    int64_t bcol0, const uint32_t *pk)
{
    if (arow >= p.rows_a)
        return;
    __nv_bfloat16 *y = reinterpret_cast<__nv_bfloat16 *>(p.y);
#pragma unroll
    for (int j = 0; j < BN; ++j) {
        const int64_t m = bcol0 + j;
        if (m < p.rows_b)
            y[m * p.ldy + arow] = bf16_half(pk[j / 2], j & 1);
    }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSFA,
                      const __grid_constant__ CUtensorMap tmSFB,
                      const __grid_constant__ CUtensorMap tmY, const GemmParams p)
{
    using C = Cfg<BN>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((smem_u32(smem) & 1023u) != 0) { // the swizzled operand tiles need 1024-B alignment
        if (threadIdx.x == 0)
            atomicExch(p.status, (int)NVFP4_ERR_CUDA);
        return;
    }
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *sf_full = empty_bar + C::kStages;
    uint64_t *sf_empty = sf_full + C::kSfSlots;
    uint64_t *acc_full = sf_empty + C::kSfSlots;
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
        for (int s = 0; s < C::kSfSlots; ++s) {
            mbar_init(&sf_full[s], 4);
            mbar_init(&sf_empty[s], 1);
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
    } else if (warp >= 6) {
        // ------------------------------- scale-factor feeders -----------------------
        const int q = warp & 3; // the TMEM lane quarter this warp may write
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
            const int split = (int)(u / tiles_ab);
            const int k0 = split * p.kt_per_split;
            const int k1 = min(p.kt_total, k0 + p.kt_per_split);
            for (int kt = k0; kt < k1; ++kt) {
                if (!mbar_wait(&full_bar[stage], phase, kWaitLimit) ||
                    !mbar_wait(&sf_empty[slot], sphase ^ 1, kWaitLimit)) {
                    if (lane == 0)
                        set_timeout(p.status);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ssfa = smem_u32(smem + C::kOffSfa + stage * C::kSfaBytes);
                const uint32_t ssfb = smem_u32(smem + C::kOffSfb + stage * C::kSfbBytes);
                const uint32_t tslot =
                    tmem + ((uint32_t)(q * 32) << 16) + C::kSfCol + slot * C::kSlotCols;
                // SFA: atom kb -> columns 4*kb .. 4*kb+3 (row r of the atom in lane r)
                uint32_t ra[16];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint4 w = lds128(ssfa + kb * 512 + lane * 16);
                    ra[4 * kb] = w.x;
                    ra[4 * kb + 1] = w.y;
                    ra[4 * kb + 2] = w.z;
                    ra[4 * kb + 3] = w.w;
                }
                tmem_st_32x32b_x16(tslot, ra);
                // SFB: atom (band h, kb) -> columns 16 + kb*kSfbColsPerKb + 4*h
#pragma unroll
                for (int h = 0; h < C::kSfbBands; ++h) {
                    uint32_t rb[16];
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint4 w = lds128(ssfb + (h * 4 + kb) * 512 + lane * 16);
                        rb[4 * kb] = w.x;
                        rb[4 * kb + 1] = w.y;
                        rb[4 * kb + 2] = w.z;
                        rb[4 * kb + 3] = w.w;
                    }
                    if constexpr (C::kSfbBands == 1) {
                        tmem_st_32x32b_x16(tslot + 16, rb);
                    } else {
                        // interleave bands: kb-major, band-minor
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            uint32_t t4[16];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                t4[i] = rb[4 * kb + i];
                            asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], "
                                         "{%1, %2, %3, %4};" ::"r"(tslot + 16 +
                                                                     kb * C::kSfbColsPerKb + 4 * h),
                                         "r"(t4[0]), "r"(t4[1]), "r"(t4[2]), "r"(t4[3])
                                         : "memory");
                        }
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sf_full[slot]);
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++slot == C::kSfSlots) {
                    slot = 0;
                    sphase ^= 1;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0, acc_phase = 0;
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
                if (!mbar_wait(&full_bar[stage], phase, kWaitLimit) ||
                    !mbar_wait(&sf_full[slot], sphase, kWaitLimit)) {
                    if (lane == 0)
                        set_timeout(p.status);
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t tsfa = tmem + C::kSfCol + slot * C::kSlotCols;
                    const uint32_t tsfb = tsfa + 16;
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
                    tc_commit(&sf_empty[slot]);
                }
                __syncwarp();
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++slot == C::kSfSlots) {
                    slot = 0;
                    sphase ^= 1;
                }
            }
            if (!ok)
                break;
            if (lane == 0)
                tc_commit(acc_full);
            __syncwarp();
            acc_phase ^= 1;
        }
        // Drain: every MMA issued by this thread completes before TMEM is freed.
        if (lane == 0) {
            tc_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0, kWaitLimit))
                set_timeout(p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue (warps 2..5) ----------------------
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
            if constexpr (BN == 256) {
                if (p.tma_store) {
                    // previous tile's bulk stores must have read the staging buffer
                    if (threadIdx.x == 64)
                        bulk_wait_group_read0();
                    named_bar_sync(1, 128);
                    stage_tile_bf16(trow, smem_u32(smem + C::kOffStaging), q * 32 + lane, alpha,
                                    [&]() {
                                        tc_fence_before();
                                        __syncwarp();
                                        if (lane == 0) // next tile's MMAs may start
                                            mbar_arrive(acc_empty);
                                    });
                    fence_proxy_async_smem();
                    named_bar_sync(1, 128);
                    if (threadIdx.x == 64) {
#pragma unroll
                        for (int b = 0; b < BN / 64; ++b)
                            tma_store_2d(&tmY, smem + C::kOffStaging + b * (BM * 128),
                                         (int)(tb * BN + b * 64), (int)(ta * BM));
                        bulk_commit_group();
                    }
                    acc_phase ^= 1;
                    continue;
                }
            }
            if (p.splits == 1 && p.out_bf16 && BN <= 128) {
                // bf16 row in registers, accumulator released before the stores
                uint32_t pk[BN / 2 > 0 ? BN / 2 : 1];
                acc_row_to_bf16<BN>(trow, alpha, pk);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(acc_empty);
                if (p.swap)
                    store_row_bf16_swap<BN>(p, arow, tb * BN, pk);
                else
                    store_row_bf16<BN>(p, arow, tb * BN, pk);
            } else {
                constexpr int NC = BN < 32 ? BN : 32;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += NC) {
                    uint32_t v[NC];
                    tmem_ld_cols<NC>(trow + c0, v);
                    tmem_ld_wait();
                    store_chunk<BN>(p, arow, tb * BN + c0, split, v, NC, alpha);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(acc_empty);
            }
            acc_phase ^= 1;
        }
    }

    if (threadIdx.x == 64)
        bulk_wait_group0(); // bulk stores complete before the CTA's shared memory goes away
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Activation of the quantizing epilogue: ACT 0 identity; ACT 1 GELU in its tanh form,
// y / (1 + exp(-2u)) with u = sqrt(2/pi) (y + 0.044715 y^3), as y * rcp(1 + 2^(y * k (1 + c y^2)))
// with k = -2 sqrt(2/pi) log2(e) and the hardware's approximate base-2 exponential and
// reciprocal (relative error ~1e-6). The exponent is clamped at 126, where the result is
// already below 1e-37 |y|: 1 + 2^126 keeps the reciprocal finite and non-zero.
__device__ __forceinline__ float fast_ex2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float fast_rcp(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

template <int ACT> __device__ __forceinline__ float epi_act(float y)
{
    if constexpr (ACT == 1) {
        const float z = y * (-2.3022082f * fmaf(0.044715f, y * y, 1.0f));
        return y * fast_rcp(1.0f + fast_ex2(fminf(z, 126.0f)));
    } else {
        return y;
    }
}

// 64 accumulator values (fp32 bits) of output row `row`, columns col..col+63 -> NVFP4:
// v = act(acc * alpha); per 16-value block sb = E4M3(bmax / t) (t = 6 sg, the quantizer's exact
// quotient), codes E2M1(v * s_rcp[sb]) with s_rcp[c] = RN(1 / RN(E4M3(c) * sg)); sb = 0 gives
// zero codes. The codes go to the row's 32-byte run, the four scales (one 64-column atom row)
// to the swizzled layout in one 4-byte store. Rows past M and columns past N hold zeros (their
// operands are TMA zero fill), so the swizzled padding of the last band and atom is written as
// zero scales.
template <int ACT>
__device__ __forceinline__ void quantize_out_chunk(const GemmParams &p, const uint32_t (&v)[64],
                                                   int64_t row, int64_t col, float alpha, float t,
                                                   float rt, const float *s_rcp)
{
    uint32_t cw[8];
    uint32_t sw = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float y[16];
        float bmax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            y[j] = epi_act<ACT>(__fmul_rn(__uint_as_float(v[16 * b + j]), alpha));
            bmax = fmaxf(bmax, fabsf(y[j]));
        }
        const uint32_t sb = t > 0.0f ? e4m3_of_quotient(bmax, t, rt) : 0u;
        const float r = s_rcp[sb]; // sb = 0: every code is 0 (selected below)
#pragma unroll
        for (int j = 0; j < 16; ++j)
            y[j] = __fmul_rn(y[j], r);
        const uint32_t lo = cvt_e2m1x8(y), hi = cvt_e2m1x8(y + 8);
        cw[2 * b] = sb != 0u ? lo : 0u;
        cw[2 * b + 1] = sb != 0u ? hi : 0u;
        sw |= sb << (8 * b);
    }
    if (row < p.rows_a && col < p.rows_b) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.q_codes + row * (p.rows_b / 2) + col / 2);
        dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        if (col + 32 < p.rows_b)
            dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    }
    const int64_t atom = col / 64;
    if (row < p.q_rows_pad && atom < p.q_apb)
        *reinterpret_cast<uint32_t *>(p.q_sf + ((row >> 7) * p.q_apb + atom) * 512 +
                                      16 * (row & 31) + 4 * ((row & 127) >> 5)) = sw;
}

// One thread's 256-column accumulator row (TMEM address trow, row r of the CTA's 128) of
// output row `row`, columns col0.. -> NVFP4. Columns 128..255 are first copied to the staging
// tile as fp32 (column-major in 16-byte groups: a warp's stores and loads are conflict-free,
// and each thread reads back only its own row), columns 0..127 are quantized from TMEM, then
// the accumulator is handed back (release()) and the saved half is quantized while the next
// tile's MMAs run.
template <int ACT, typename Release>
__device__ __forceinline__ void quantize_out_row(const GemmParams &p, uint32_t trow, uint32_t tpark,
                                                 uint32_t stg, int r, int64_t row, int64_t col0,
                                                 float alpha, float t, float rt,
                                                 const float *s_rcp, Release release)
{
    // the accumulator is handed back as soon as it is copied: columns 128-255 to the staging
    // tile (fp32), columns 0-127 to TMEM columns the MMAs do not use (tpark); the activation and
    // the quantization of the whole tile then overlap the next tile's MMAs
#pragma unroll 1
    for (int c0 = 128; c0 < 256; c0 += 64) {
        uint32_t v[64];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tmem_ld_32x32b_x16(trow + c0 + 16 * i, v + 16 * i);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 16; ++g)
            sts128(stg + ((((c0 - 128) >> 2) + g) * 128 + r) * 16, v[4 * g], v[4 * g + 1],
                   v[4 * g + 2], v[4 * g + 3]);
    }
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 64) {
        uint32_t v[64];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tmem_ld_32x32b_x16(trow + c0 + 16 * i, v + 16 * i);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tmem_st_32x32b_x16(tpark + c0 + 16 * i, v + 16 * i);
    }
    tmem_st_wait();
    release();
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 64) {
        uint32_t v[64];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tmem_ld_32x32b_x16(tpark + c0 + 16 * i, v + 16 * i);
        tmem_ld_wait();
        quantize_out_chunk<ACT>(p, v, row, col0 + c0, alpha, t, rt, s_rcp);
    }
#pragma unroll 1
    for (int c0 = 128; c0 < 256; c0 += 64) {
        uint32_t v[64];
#pragma unroll
        for (int g = 0; g < 16; ++g) {
            const uint4 w = lds128(stg + ((((c0 - 128) >> 2) + g) * 128 + r) * 16);
            v[4 * g] = w.x;
            v[4 * g + 1] = w.y;
            v[4 * g + 2] = w.z;
            v[4 * g + 3] = w.w;
        }
        quantize_out_chunk<ACT>(p, v, row, col0 + c0, alpha, t, rt, s_rcp);
    }
}

// ---------------------------------------------------------------------------------------
// 2-SM variant: a CTA pair (cluster of 2) computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M256 N256 K64). Each CTA loads its 128 rows of A and its 128
// rows of B, so the shared-memory traffic per SM per k-tile drops from ~108 KB (1-SM 128x256
// tile: TMA writes + MMA reads) to ~76 KB. QOUT: the epilogue quantizes the (activated) tile
// to NVFP4 with a static global scale instead of storing bf16 (quantize_out_row): the next
// layer's operand is produced without a bf16 round trip. The leader CTA (rank 0) issues the MMAs and
// commits to barriers of both CTAs; the other CTA's TMA loads of A / B and its feeder and
// epilogue warps arrive on the leader's barriers. Scale factors: each CTA's TMEM holds SFA
// of its own 128 rows and SFB of all 256 columns (its feeders write both). Only the bf16,
// un-split case uses it (TMA-store epilogue).
// ---------------------------------------------------------------------------------------

// One CTA's 128 x 256 bf16 output tile through a 32 KB staging tile (two 64-column boxes), in
// two halves: accumulator columns 0-127 are converted and their TMA store issued while columns
// 128-255 are read from TMEM; `release` follows the last TMEM read; the second half is staged
// once the first store has left the staging tile. Run by the four epilogue warps (r: this
// thread's row, TMEM lane; `issuer`: the thread that issues and tracks the stores).
// Half of the tile's writes thus leave while the MMA warp still waits for the accumulator: the
// writes that follow the release compete with the next tile's operand loads.
template <typename Release>
__device__ __forceinline__ void stage_store_tile_halves(const GemmParams &p, const CUtensorMap *tmY,
                                                        uint8_t *stg, uint32_t trow, int r,
                                                        float alpha, bool issuer, int64_t yrow,
                                                        int64_t ycol, Release release)
{
    const uint32_t s = smem_u32(stg);
    auto store = [&](int half) {
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
            // boxes that start past the last row or column of Y hold nothing to store
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int64_t col = ycol + (2 * half + b) * 64;
                if (yrow < p.rows_a && col < p.rows_b)
                    tma_store_2d(tmY, stg + b * (128 * 128), (int)col, (int)yrow);
            }
            bulk_commit_group();
        }
    };
    uint32_t va[64], vb[64];
    tmem_ld_64cols(trow, va);
    tmem_ld_wait();
    tmem_ld_64cols(trow + 64, vb);
    stage_box_bf16(va, s, 0, r, alpha);
    tmem_ld_wait();
    stage_box_bf16(vb, s, 1, r, alpha);
    tmem_ld_64cols(trow + 128, va);
    tmem_ld_64cols(trow + 192, vb);
    store(0);
    tmem_ld_wait();
    release();
    if (issuer)
        bulk_wait_group_read0(); // the first half has left the staging tile
    named_bar_sync(1, 128);
    stage_box_bf16(va, s, 0, r, alpha);
    stage_box_bf16(vb, s, 1, r, alpha);
    store(1);
}

// Shared-memory and TMEM layout of the pair kernel. bf16 output: five operand stages and a 32 KB
// bf16 staging tile (the output leaves in two halves), four scale slots; quantizing epilogue:
// four stages and 64 KB of staging (fp32 columns 128-255 of each row), two scale slots and 128
// TMEM columns for columns 0-127 (both kept while the tile is quantized after the hand-back).
template <bool QOUT> struct Pair {
    static constexpr int kStages = QOUT ? 4 : 5;
    static constexpr int kABytes = 128 * 128;     // this CTA's 128 rows of A
    static constexpr int kBBytes = 128 * 128;     // this CTA's 128 rows of B
    static constexpr int kSfaBytes = 4 * 512;     // SFA atoms of this CTA's rows
    static constexpr int kSfbBytes = 2 * 4 * 512; // SFB atoms of all 256 columns
    static constexpr int kOffB = kStages * kABytes;
    static constexpr int kOffSfa = kOffB + kStages * kBBytes;
    static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
    static constexpr int kOffStaging = kOffSfb + kStages * kSfbBytes;
    static constexpr int kStagingBytes = QOUT ? 128 * 128 * 4 : 128 * 128 * 2;
    static constexpr int kOffBar = kOffStaging + kStagingBytes;
    static constexpr int kOffRcp = kOffBar + 512; // quantizing epilogue: 128 reciprocals
    static constexpr int kSmemBytes = kOffRcp + 512;
    static constexpr uint32_t kTxAB = 2 * (kABytes + kBBytes); // both CTAs, on the leader
    static constexpr uint32_t kTxSf = kSfaBytes + kSfbBytes;   // own CTA
    // quantizing epilogue: two scale slots, so that 128 TMEM columns after them can hold half of
    // the accumulator while its tile is quantized (quantize_out_row)
    static constexpr int kSfSlots = QOUT ? 2 : 4;
    static constexpr int kSlotCols = 16 + 32; // SFA 4 x 4, SFB 4 x 8
    static constexpr int kSfCol = 256;
    static constexpr int kParkCol = kSfCol + kSfSlots * kSlotCols; // QOUT: columns 0-127 kept
    static constexpr int kTmemCols = 512;
    static constexpr uint32_t kIdesc =
        (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
    // low-rank k-tiles: kind::f16 with D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9 and
    // 10-12 = 1), K-major, M256 x N256; a 64-wide bf16 k-tile fills the same 128-byte smem
    // rows as a 256-wide FP4 k-tile, so it reuses the stage buffers and their byte counts
    static constexpr uint32_t kIdescLr = (1u << 4) | (1u << 7) | (1u << 10) |
                                         ((uint32_t)(256 >> 3) << 17) |
                                         ((uint32_t)(256 >> 4) << 24);
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kOffStaging % 1024 == 0, "swizzled staging alignment");
    static_assert(kSfCol + kSfSlots * kSlotCols <= kTmemCols, "TMEM budget");
    static_assert(!QOUT || kParkCol + 128 <= kTmemCols, "TMEM budget of the parked columns");
};

// 2-SM bf16 MMA issued by the leader CTA (the low-rank k-tiles): D (+)= A x B^T, fp32.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

template <bool QOUT, bool LR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFA,
                           const __grid_constant__ CUtensorMap tmSFB,
                           const __grid_constant__ CUtensorMap tmY,
                           const __grid_constant__ CUtensorMap tmT,
                           const __grid_constant__ CUtensorMap tmU, const GemmParams p)
{
    using C = Pair<QOUT>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0)
            atomicExch(p.status, (int)NVFP4_ERR_CUDA);
        return; // uniform across the cluster: both CTAs see the same layout
    }
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kOffBar); // leader only
    uint64_t *sfdata = full_bar + C::kStages;                            // own SF TMA
    uint64_t *empty_bar = sfdata + C::kStages;                           // both
    uint64_t *sf_full = empty_bar + C::kStages;                          // leader only
    uint64_t *sf_empty = sf_full + C::kSfSlots;                          // both
    uint64_t *acc_full = sf_empty + C::kSfSlots;                         // both
    uint64_t *acc_empty = acc_full + 1;                                  // leader only
    uint64_t *drain_bar = acc_full + 2;                                  // leader only
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 3);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&sfdata[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < C::kSfSlots; ++s) {
            mbar_init(&sf_full[s], 8); // four feeder warps in each CTA
            mbar_init(&sf_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8); // four epilogue warps in each CTA
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

    const int64_t tiles_ab = p.tiles_a * p.tiles_b; // tiles_a counts 256-row pairs
    const int64_t cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int kt_tile = p.kt_total + (LR ? p.lr_kt : 0); // stage uses per tile

    if (warp == 0) {
        // ------------------------------- TMA producer (both CTAs) ---------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmSFA);
            tma_prefetch_desc(&tmSFB);
            if constexpr (LR) {
                tma_prefetch_desc(&tmT);
                tma_prefetch_desc(&tmU);
            }
            pdl_wait(); // operands come from the stream's earlier kernels
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t u = cluster_id; u < tiles_ab && ok; u += nclusters) {
                const int64_t ta = u % p.tiles_a, tb = u / p.tiles_a;
                const int arow = (int)(ta * 256 + rank * 128);
                const int brow = (int)(tb * 256 + rank * 128);
                for (int kt = 0; kt < kt_tile; ++kt) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kWaitLimit)) {
                        set_timeout(p.status);
                        ok = false;
                        break;
                    }
                    const uint32_t leader_full = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (leader)
                        mbar_arrive_expect_tx(&full_bar[stage], C::kTxAB);
                    if (LR && kt >= p.kt_total) {
                        // low-rank k-tile: 64 ranks of T' (A side) and U (B side), 16 KB each;
                        // no scales, and sfdata[stage] is left alone: its phases count the
                        // stage's FP4 uses only (the feeders track them per stage)
                        const int x = (kt - p.kt_total) * 64;
                        tma_load_2d_pair(smem + stage * C::kABytes, &tmT, leader_full, x, arow);
                        tma_load_2d_pair(smem + C::kOffB + stage * C::kBBytes, &tmU, leader_full,
                                         x, brow);
                        if (++stage == C::kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                        continue;
                    }
                    mbar_arrive_expect_tx(&sfdata[stage], C::kTxSf);
                    tma_load_2d_pair(smem + stage * C::kABytes, &tmA, leader_full, kt * 128, arow);
                    tma_load_2d_pair(smem + C::kOffB + stage * C::kBBytes, &tmB, leader_full,
                                     kt * 128, brow);
                    tma_load_3d(smem + C::kOffSfa + stage * C::kSfaBytes, &tmSFA, &sfdata[stage], 0,
                                kt * 4, arow >> 7);
                    tma_load_3d(smem + C::kOffSfb + stage * C::kSfbBytes, &tmSFB, &sfdata[stage], 0,
                                kt * 4, (int)(tb * 2));
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp >= 6) {
        // ------------------------------- scale-factor feeders (both CTAs) -------------
        const int q = warp & 3;
        const uint32_t leader_sf_full0 = mapa_shared(smem_u32(&sf_full[0]), 0);
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        // LR: per-stage parity of sfdata, which completes a phase per FP4 use of the stage
        // only. The next FP4 use of a stage is armed after the MMA warp has consumed this one
        // (which needs these warps' slot), so sfdata never runs two phases ahead of them.
        uint32_t sfbits = 0;
        bool ok = true;
        for (int64_t u = cluster_id; u < tiles_ab && ok; u += nclusters) {
            for (int kt = 0; kt < kt_tile; ++kt) {
                if (LR && kt >= p.kt_total) { // low-rank k-tile: no scales to feed
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                    continue;
                }
                const uint32_t sfpar = LR ? ((sfbits >> stage) & 1u) : phase;
                if (LR)
                    sfbits ^= 1u << stage;
                if (!mbar_wait(&sfdata[stage], sfpar, kWaitLimit) ||
                    !mbar_wait(&sf_empty[slot], sphase ^ 1, kWaitLimit)) {
                    if (lane == 0)
                        set_timeout(p.status);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ssfa = smem_u32(smem + C::kOffSfa + stage * C::kSfaBytes);
                const uint32_t ssfb = smem_u32(smem + C::kOffSfb + stage * C::kSfbBytes);
                const uint32_t tslot =
                    tmem + ((uint32_t)(q * 32) << 16) + C::kSfCol + slot * C::kSlotCols;
                uint32_t ra[16];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint4 w = lds128(ssfa + kb * 512 + lane * 16);
                    ra[4 * kb] = w.x;
                    ra[4 * kb + 1] = w.y;
                    ra[4 * kb + 2] = w.z;
                    ra[4 * kb + 3] = w.w;
                }
                tmem_st_32x32b_x16(tslot, ra);
                // SFB: atom (band h, kb) -> columns 16 + 8*kb + 4*h
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    uint32_t rb[16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 w = lds128(ssfb + (h * 4 + kb) * 512 + lane * 16);
                        rb[4 * h] = w.x;
                        rb[4 * h + 1] = w.y;
                        rb[4 * h + 2] = w.z;
                        rb[4 * h + 3] = w.w;
                    }
                    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], "
                                 "{%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(tslot + 16 + 8 * kb),
                                 "r"(rb[0]), "r"(rb[1]), "r"(rb[2]), "r"(rb[3]), "r"(rb[4]),
                                 "r"(rb[5]), "r"(rb[6]), "r"(rb[7])
                                 : "memory");
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_remote(leader_sf_full0 + 8 * slot);
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++slot == C::kSfSlots) {
                    slot = 0;
                    sphase ^= 1;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer (leader) ---------------------------
        if (leader) {
            int stage = 0, slot = 0;
            uint32_t phase = 0, sphase = 0, acc_phase = 0;
            bool ok = true;
            for (int64_t u = cluster_id; u < tiles_ab && ok; u += nclusters) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1, kWaitLimit)) {
                    if (lane == 0)
                        set_timeout(p.status);
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < kt_tile; ++kt) {
                    if (LR && kt >= p.kt_total) {
                        if (!mbar_wait(&full_bar[stage], phase, kWaitLimit)) {
                            if (lane == 0)
                                set_timeout(p.status);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (lane == 0) {
                            const uint64_t adesc = smem_desc(smem_u32(smem + stage * C::kABytes),
                                                             16, 1024, kLayoutSwizzle128B);
                            const uint64_t bdesc =
                                smem_desc(smem_u32(smem + C::kOffB + stage * C::kBBytes), 16,
                                          1024, kLayoutSwizzle128B);
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb) // K16 bf16 = 32 bytes per MMA
                                tc_mma_bf16_pair(tmem, adesc + (uint64_t)(2 * kb),
                                                 bdesc + (uint64_t)(2 * kb), C::kIdescLr,
                                                 (kt > 0 || kb > 0) ? 1u : 0u);
                            tc_commit_pair_mc(&empty_bar[stage], 0x3);
                        }
                        __syncwarp();
                        if (++stage == C::kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                        continue;
                    }
                    if (!mbar_wait(&full_bar[stage], phase, kWaitLimit) ||
                        !mbar_wait(&sf_full[slot], sphase, kWaitLimit)) {
                        if (lane == 0)
                            set_timeout(p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t tsfa = tmem + C::kSfCol + slot * C::kSlotCols;
                        const uint32_t tsfb = tsfa + 16;
                        const uint64_t adesc = smem_desc(smem_u32(smem + stage * C::kABytes), 16,
                                                         1024, kLayoutSwizzle128B);
                        const uint64_t bdesc =
                            smem_desc(smem_u32(smem + C::kOffB + stage * C::kBBytes), 16, 1024,
                                      kLayoutSwizzle128B);
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb)
                            tc_mma_nvf4_pair(tmem, adesc + (uint64_t)(2 * kb),
                                             bdesc + (uint64_t)(2 * kb), C::kIdesc, tsfa + kb * 4,
                                             tsfb + kb * 8, (kt > 0 || kb > 0) ? 1u : 0u);
                        tc_commit_pair_mc(&empty_bar[stage], 0x3);
                        tc_commit_pair_mc(&sf_empty[slot], 0x3);
                    }
                    __syncwarp();
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                    if (++slot == C::kSfSlots) {
                        slot = 0;
                        sphase ^= 1;
                    }
                }
                if (!ok)
                    break;
                if (lane == 0)
                    tc_commit_pair_mc(acc_full, 0x3);
                __syncwarp();
                acc_phase ^= 1;
            }
            if (lane == 0) {
                tc_commit_pair(drain_bar);
                if (!mbar_wait(drain_bar, 0, kWaitLimit))
                    set_timeout(p.status);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------- epilogue (both CTAs, warps 2..5) -------------
        const int q = warp & 3;
        pdl_wait(); // global scales (and Y's previous readers) belong to earlier kernels
        float alpha = __fmul_rn(*p.a_gs, *p.w_gs);
        if (LR && alpha == 0.0f)
            alpha = 1.0f; // the FP4 product is zero; T' was not divided either
        const uint32_t leader_acc_empty = mapa_shared(smem_u32(acc_empty), 0);
        uint32_t acc_phase = 0;
        float q_t = 0.0f, q_rt = 0.0f;
        float *s_rcp = reinterpret_cast<float *>(smem + C::kOffRcp);
        if constexpr (QOUT) {
            const float sg = __fdiv_rn(*p.q_amax, 2688.0f); // 6 * 448, as the quantizer
            q_t = __fmul_rn(sg, 6.0f);
            q_rt = __frcp_rn(q_t);
            const int i = (int)threadIdx.x - 64; // 0..127
            s_rcp[i] = __frcp_rn(__fmul_rn(e4m3_to_f32((uint32_t)i), sg));
            if (i == 0 && blockIdx.x == 0)
                *p.q_gs = sg;
            named_bar_sync(1, 128);
        }
        for (int64_t u = cluster_id; u < tiles_ab; u += nclusters) {
            const int64_t ta = u % p.tiles_a, tb = u / p.tiles_a;
            if (!mbar_wait(acc_full, acc_phase, kWaitLimit)) {
                if (lane == 0)
                    set_timeout(p.status);
                break;
            }
            tc_fence_after();
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
            if constexpr (QOUT) {
                auto release = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_remote(leader_acc_empty); // this CTA's accumulator is read
                };
                const uint32_t stg = smem_u32(smem + C::kOffStaging);
                const int64_t row = ta * 256 + rank * 128 + q * 32 + lane;
                const uint32_t tpark = trow + C::kParkCol;
                if (p.act == 1)
                    quantize_out_row<1>(p, trow, tpark, stg, q * 32 + lane, row, tb * 256, alpha,
                                        q_t, q_rt, s_rcp, release);
                else
                    quantize_out_row<0>(p, trow, tpark, stg, q * 32 + lane, row, tb * 256, alpha,
                                        q_t, q_rt, s_rcp, release);
                acc_phase ^= 1;
                continue;
            }
            if (threadIdx.x == 64)
                bulk_wait_group_read0(); // the previous tile's second half has left the staging
            named_bar_sync(1, 128);
            stage_store_tile_halves(p, &tmY, smem + C::kOffStaging, trow, q * 32 + lane, alpha,
                                    threadIdx.x == 64, ta * 256 + rank * 128, tb * 256, [&]() {
                                        tc_fence_before();
                                        __syncwarp();
                                        if (lane == 0)
                                            mbar_arrive_remote(leader_acc_empty); // read
                                    });
            acc_phase ^= 1;
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
// Small M (<= 128, swap-AB): one 128-row tile of W per thread-block cluster, its K range
// split over the cluster's csplit CTAs. Each CTA streams its share of k-tiles through the
// same warp-specialized pipeline as the persistent kernel (TMA producer, scale-factor
// feeders, MMA issuer, epilogue), sized so that two CTAs fit on an SM. CTAs 1.. stage their
// fp32 partial accumulators in their own (drained) shared memory; the leader (rank 0) adds
// them to its own in rank order through distributed shared memory, scales and stores. So
// every SM streams weights, with no workspace and no second kernel, and the sum order is
// fixed. The kernel takes part in programmatic dependent launch: its set-up overlaps the
// previous kernel of the stream, its global reads and writes wait for that kernel.
// ---------------------------------------------------------------------------------------

// Fused-activation layout (M <= 32): the TMA ring carries W and its scales only; the
// activations' codes (B operand, 128B-swizzled, one BN x 128-byte tile per k-tile) and scale
// atoms (2 KB per k-tile) of this CTA's k-range (at most kXqMaxKt k-tiles) stay resident,
// written by the CTA itself from the bf16 / fp32 activations.
constexpr int kXqMaxKt = 8;
template <int BN> struct XqLayout {
    static constexpr int kStages = BN <= 16 ? 4 : 3;
    static constexpr int kSfbBands = 1;
    static constexpr int kABytes = BM * 128;
    static constexpr int kBBytes = BN * 128; // per resident k-tile
    static constexpr int kSfaBytes = 4 * 512;
    static constexpr int kSfbBytes = 4 * 512; // per resident k-tile
    static constexpr int kOffSfa = kStages * kABytes;
    static constexpr int kOffB = kOffSfa + kStages * kSfaBytes; // resident B
    static constexpr int kOffSfb = kOffB + kXqMaxKt * kBBytes;   // resident SFB atoms
    static constexpr int kOffBar = kOffSfb + kXqMaxKt * kSfbBytes;
    static constexpr int kSmemBytes = kOffBar + 512;
    static constexpr uint32_t kTx = kABytes + kSfaBytes; // per stage: W tile and its scales
    static constexpr int kAccCols = BN < 32 ? 32 : BN;
    static constexpr int kSfSlots = 4;
    static constexpr int kSfbColsPerKb = 4;
    static constexpr int kSlotCols = 32;
    static constexpr int kSfCol = kAccCols;
    static constexpr int kUsedCols = kSfCol + kSfSlots * kSlotCols;
    static constexpr int kTmemCols = kUsedCols <= 128 ? 128 : 256;
    static constexpr uint32_t kIdesc =
        (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static constexpr bool kResidentB = true;
    static_assert(kOffB % 1024 == 0, "swizzled operand alignment");
};

template <int BN, bool XQ = false> struct SmallCfg {
    // stages that keep one CTA at <= 113 KB of shared memory (two per SM)
    static constexpr int kStages = BN <= 16 ? 5 : BN <= 64 ? 4 : 3;
    using L = typename std::conditional<XQ, XqLayout<BN>, Cfg<BN, kStages>>::type;
    static_assert(L::kSmemBytes <= 115712, "two CTAs per SM");
    static_assert(L::kTmemCols <= 256, "two CTAs per SM");
    // partial accumulators of a non-leader CTA, [BN][128] fp32, over the drained stages
    static_assert(BN * 128 * 4 + BN * 128 * 2 <= L::kOffSfa,
                  "partials and bf16 output staging fit in the operand stages");
};



struct SmallParams {
    int64_t rows_a, rows_b; // weight rows (N), activation rows (M)
    int kt_total;           // 256-wide k-tiles
    int csplit;             // CTAs per cluster = K splits
    const float *a_gs, *w_gs;
    void *y;
    int64_t ldy; // = N
    int out_bf16;
    int tma_store;  // 1: each CTA stages its slice of the output tile, one TMA store writes it
    int resident_w; // 1: W is not written by earlier work still running on the stream, so
                    // its first stages load before the programmatic-launch wait
    int *status;
    // fused activation quantize (XQ kernels): x [M x K] row-major, bf16 (x_bf16) or fp32;
    // x_gs_out (may be null): receives the activations' global scale
    const void *x;
    int x_bf16;
    int64_t K;
    float *x_gs_out;
};

// Output rows [rank*BN/CS, (rank+1)*BN/CS) of the tile, summed over the CS partials of the
// cluster in rank order (the same order on every CTA), scaled, cast and stored. Thread t owns
// output column n = 128*ta + t. Remote loads are issued in batches of up to 32 so that one
// distributed-shared-memory round trip serves a batch. bf16 results are staged after the
// partials, fp32 results overwrite this CTA's own slice rows (each thread rewrites exactly the
// elements it read; peers never read this CTA's slice), then one TMA store writes the
// [BN/CS x 128] box (clipped at M and N). With CS > 1 the caller waits on the cluster barrier
// this function arrives on once its remote reads are done, before the CTA may exit.
template <int BN, int CS>
__device__ __forceinline__ void reduce_slice(const SmallParams &p, uint8_t *smem, uint32_t rank,
                                             int t, int64_t ta, float alpha,
                                             const CUtensorMap *tmY)
{
    constexpr int SR = BN / CS;                         // output rows of this CTA
    constexpr int RB = (32 / CS) < SR ? (32 / CS) : SR; // rows per batch
    static_assert(BN % CS == 0 && SR % RB == 0, "slice shape");
    const int m0 = (int)rank * SR;
    const uint32_t col = smem_u32(smem) + (uint32_t)t * 4u;
    uint32_t src[CS];
#pragma unroll
    for (int j = 0; j < CS; ++j)
        src[j] = CS == 1 ? col : mapa_shared(col, (uint32_t)j);
    float *part = reinterpret_cast<float *>(smem);
    __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(smem + BN * BM * 4);
    const int64_t n = ta * BM + t;
#pragma unroll 1
    for (int mb = 0; mb < SR; mb += RB) {
        float v[RB][CS];
#pragma unroll
        for (int rr = 0; rr < RB; ++rr) {
            const uint32_t off = (uint32_t)(m0 + mb + rr) * (BM * 4);
#pragma unroll
            for (int j = 0; j < CS; ++j) {
                if constexpr (CS == 1)
                    v[rr][j] = part[(m0 + mb + rr) * BM + t];
                else
                    v[rr][j] = ld_shared_cluster_f32(src[j] + off);
            }
        }
#pragma unroll
        for (int rr = 0; rr < RB; ++rr) {
            float acc = v[rr][0];
#pragma unroll
            for (int j = 1; j < CS; ++j)
                acc += v[rr][j];
            const float r = acc * alpha;
            const int m = m0 + mb + rr;
            if (p.tma_store) {
                if (p.out_bf16)
                    ob[(mb + rr) * BM + t] = __float2bfloat16_rn(r);
                else
                    part[m * BM + t] = r;
            } else if (m < p.rows_b && n < p.rows_a) {
                if (p.out_bf16)
                    reinterpret_cast<__nv_bfloat16 *>(p.y)[m * p.ldy + n] = __float2bfloat16_rn(r);
                else
                    reinterpret_cast<float *>(p.y)[m * p.ldy + n] = r;
            }
        }
    }
    if constexpr (CS > 1) {
        __syncwarp();
        cluster_arrive(); // done reading the other CTAs' partials (waited on before exit)
    }
    if (p.tma_store) {
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (t == 0 && m0 < p.rows_b) {
            const void *src_tile = p.out_bf16 ? static_cast<const void *>(ob)
                                              : static_cast<const void *>(part + m0 * BM);
            tma_store_2d(tmY, src_tile, (int)(ta * BM), m0);
            bulk_commit_group();
            bulk_wait_group_read0(); // shared memory is read before the CTA may exit
        }
    }
}


// Fused activation quantize of the XQ kernels, run by every thread of the CTA before its
// warp roles: max |x| over the whole M x K activation tensor (each CTA of the cluster folds a
// share, the shares are combined through distributed shared memory, so every cluster holds
// the same exact maximum), sg = amax / 2688, and this CTA's k-range of x encoded into the
// resident B tiles (codes, 128B-swizzled rows, the layout TMA would write) and scale atoms,
// with the quantizer's arithmetic (the codes equal nvfp4_quantize's). Rows M .. BN-1 and
// blocks past K stay zero. Returns sg.
template <int BN, typename L>
__device__ __forceinline__ float xq_prologue(const SmallParams &p, uint8_t *smem, uint32_t rank,
                                             int cs, int k0, int k1)
{
    __shared__ float s_warp[kThreads / 32];
    __shared__ float s_part; // this CTA's share of the maximum (read by the cluster)
    __shared__ float s_sg;
    __shared__ float s_rcp[128];
    const int tid = threadIdx.x;
    const int nk = k1 - k0;
    // zero the resident operand region of this CTA's k-tiles
    {
        uint4 *zb = reinterpret_cast<uint4 *>(smem + L::kOffB);
        const int nb16 = nk * L::kBBytes / 16;
        for (int i = tid; i < nb16; i += kThreads)
            zb[i] = make_uint4(0u, 0u, 0u, 0u);
        uint4 *zs = reinterpret_cast<uint4 *>(smem + L::kOffSfb);
        const int ns16 = nk * L::kSfbBytes / 16;
        for (int i = tid; i < ns16; i += kThreads)
            zs[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    // max |x| over this CTA's share of the tensor (16-byte vectors)
    const int64_t nvec = p.rows_b * p.K * (p.x_bf16 ? 2 : 4) / 16;
    const int64_t v0 = nvec * rank / cs, v1 = nvec * (rank + 1) / cs;
    const uint4 *xv = reinterpret_cast<const uint4 *>(p.x);
    float m = 0.0f;
    constexpr int kVin = 8; // loads in flight per thread
    for (int64_t i0 = v0 + tid; i0 < v1; i0 += (int64_t)kThreads * kVin) {
        uint4 w[kVin];
#pragma unroll
        for (int q = 0; q < kVin; ++q) {
            const int64_t i = i0 + (int64_t)q * kThreads;
            w[q] = i < v1 ? __ldg(xv + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < kVin; ++q) {
            const uint32_t u[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (p.x_bf16)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(u[j] << 16)),
                                       fabsf(__uint_as_float(u[j] & 0xFFFF0000u))));
                else
                    m = fmaxf(m, fabsf(__uint_as_float(u[j])));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((tid & 31) == 0)
        s_warp[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
        float f = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w)
            f = fmaxf(f, s_warp[w]);
        s_part = f;
    }
    if (cs > 1)
        cluster_sync(); // every share of the cluster is in place
    else
        __syncthreads();
    if (tid == 0) {
        float amax = s_part;
        for (int r = 0; r < cs; ++r)
            if (r != (int)rank)
                amax = fmaxf(amax, ld_shared_cluster_f32(mapa_shared(smem_u32(&s_part), r)));
        const float sg = __fdiv_rn(amax, 2688.0f); // 6 * 448
        s_sg = sg;
        if (blockIdx.x == 0 && p.x_gs_out)
            *p.x_gs_out = sg;
    }
    __syncthreads();
    const float sg = s_sg;
    const float t = __fmul_rn(sg, 6.0f);
    const float rt = __frcp_rn(t);
    if (tid < 128)
        s_rcp[tid] = __frcp_rn(__fmul_rn(e4m3_to_f32(tid), sg));
    __syncthreads();
    // encode rows 0 .. M-1 of k-tiles k0 .. k1-1, two 16-value blocks per thread step (both
    // blocks' loads in flight together)
    const int nbk = (int)(p.K >> 4); // blocks per row
    const int total = (int)p.rows_b * nk * 16;
    const uint8_t *xb = reinterpret_cast<const uint8_t *>(p.x);
    const int esz = p.x_bf16 ? 2 : 4;
    auto locate = [&](int i, int &r, int &j, int &bb, int &kb) {
        bb = i & 15;          // block inside the k-tile
        j = (i >> 4) % nk;    // resident k-tile
        r = (i >> 4) / nk;    // row
        kb = (k0 + j) * 16 + bb; // block along K
    };
    auto load_block = [&](int r, int kb, uint4 (&raw)[4]) {
        const uint4 *src =
            reinterpret_cast<const uint4 *>(xb + ((int64_t)r * p.K + kb * 16) * esz);
        raw[0] = __ldg(src);
        raw[1] = __ldg(src + 1);
        if (!p.x_bf16) {
            raw[2] = __ldg(src + 2);
            raw[3] = __ldg(src + 3);
        }
    };
    auto encode_block = [&](int r, int j, int bb, const uint4 (&raw)[4]) {
        float v[16];
        if (p.x_bf16) {
            const uint32_t u[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w,
                                   raw[1].x, raw[1].y, raw[1].z, raw[1].w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                v[2 * q] = __uint_as_float(u[q] << 16);
                v[2 * q + 1] = __uint_as_float(u[q] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[4 * q] = __uint_as_float(raw[q].x);
                v[4 * q + 1] = __uint_as_float(raw[q].y);
                v[4 * q + 2] = __uint_as_float(raw[q].z);
                v[4 * q + 3] = __uint_as_float(raw[q].w);
            }
        }
        float bm = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q)
            bm = fmaxf(bm, fabsf(v[q]));
        const uint32_t sb = sg > 0.0f ? e4m3_of_quotient(bm, t, rt) : 0u;
        if (sb == 0u)
            return; // codes and scale stay zero
        const float rcp = s_rcp[sb];
        float y[16];
#pragma unroll
        for (int q = 0; q < 16; q += 2) {
            const float2 pr = __fmul2_rn(make_float2(v[q], v[q + 1]), make_float2(rcp, rcp));
            y[q] = pr.x;
            y[q + 1] = pr.y;
        }
        const uint2 codes = make_uint2(cvt_e2m1x8(y), cvt_e2m1x8(y + 8));
        // B tile j: row r at r * 128 bytes, 16-byte chunk c stored at c ^ (r % 8)
        uint8_t *bt = smem + L::kOffB + j * L::kBBytes + r * 128;
        *reinterpret_cast<uint2 *>(bt + (((bb >> 1) ^ (r & 7)) << 4) + (bb & 1) * 8) = codes;
        // scale atom (r, bb) of k-tile j
        smem[L::kOffSfb + j * L::kSfbBytes + (bb >> 2) * 512 + 16 * (r & 31) +
             4 * ((r & 127) >> 5) + (bb & 3)] = (uint8_t)sb;
    };
    for (int i = tid; i < total; i += 2 * kThreads) {
        const int i2 = i + kThreads;
        int r0, j0, bb0, kb0, r1 = 0, j1 = 0, bb1 = 0, kb1 = nbk;
        locate(i, r0, j0, bb0, kb0);
        if (i2 < total)
            locate(i2, r1, j1, bb1, kb1);
        uint4 raw0[4], raw1[4];
        if (kb0 < nbk)
            load_block(r0, kb0, raw0);
        if (kb1 < nbk)
            load_block(r1, kb1, raw1);
        if (kb0 < nbk)
            encode_block(r0, j0, bb0, raw0);
        if (kb1 < nbk)
            encode_block(r1, j1, bb1, raw1);
    }
    fence_proxy_async_smem(); // the tensor cores read the B tiles through the async proxy
    __syncthreads();
    return sg;
}

template <int BN, bool XQ>
__global__ void __launch_bounds__(kThreads, 2)
    nvfp4_gemm_smallm_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmSFA,
                             const __grid_constant__ CUtensorMap tmSFB,
                             const __grid_constant__ CUtensorMap tmY, const SmallParams p)
{
    using C = typename SmallCfg<BN, XQ>::L;
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((smem_u32(smem) & 1023u) != 0) { // same for every CTA: the whole grid returns here
        if (threadIdx.x == 0)
            atomicExch(p.status, (int)NVFP4_ERR_CUDA);
        return;
    }
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *sf_full = empty_bar + C::kStages;
    uint64_t *sf_empty = sf_full + C::kSfSlots;
    uint64_t *acc_full = sf_empty + C::kSfSlots;
    uint64_t *drain_bar = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cs = p.csplit;
    const uint32_t rank = cs > 1 ? cluster_ctarank() : 0u;
    const int64_t ta = blockIdx.x / cs;
    const int k0 = (int)((int64_t)rank * p.kt_total / cs);
    const int k1 = (int)((int64_t)(rank + 1) * p.kt_total / cs);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < C::kSfSlots; ++s) {
            mbar_init(&sf_full[s], 4);
            mbar_init(&sf_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    if (cs > 1)
        cluster_sync(); // barriers initialised cluster-wide before any remote arrival
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Every CTA holds its TMEM by now, so a dependent grid's CTAs never take columns this
    // grid still has to allocate.
    pdl_launch_dependents();
    float alpha = 0.0f; // sgA * sgW, read by the epilogue warps

    // Resident weights: the first stages' W tiles and scales are requested while the
    // previous kernel may still run (the stages start out free); the activations always
    // wait for it.
    const int pre = p.resident_w ? min(k1 - k0, C::kStages) : 0;
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmSFA);
        if constexpr (!XQ) {
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmSFB);
        }
        for (int i = 0; i < pre; ++i) {
            mbar_arrive_expect_tx(&full_bar[i], C::kTx);
            tma_load_2d(smem + i * C::kABytes, &tmA, &full_bar[i], (k0 + i) * 128,
                        (int)(ta * BM));
            tma_load_3d(smem + C::kOffSfa + i * C::kSfaBytes, &tmSFA, &full_bar[i], 0,
                        (k0 + i) * 4, (int)ta);
        }
    }
    float sg_x = 0.0f; // XQ: the activations' global scale
    if constexpr (XQ) {
        pdl_wait(); // the activations may come from the previous kernel
        sg_x = xq_prologue<BN, C>(p, smem, rank, cs, k0, k1);
    }

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            pdl_wait(); // operands may come from the previous kernel
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int kt = k0; kt < k1; ++kt) {
                uint8_t *sa = smem + stage * C::kABytes;
                uint8_t *sb = smem + C::kOffB + stage * C::kBBytes;
                uint8_t *ssfa = smem + C::kOffSfa + stage * C::kSfaBytes;
                uint8_t *ssfb = smem + C::kOffSfb + stage * C::kSfbBytes;
                if (kt - k0 >= pre) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kWaitLimit)) {
                        set_timeout(p.status);
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[stage], C::kTx);
                    tma_load_2d(sa, &tmA, &full_bar[stage], kt * 128, (int)(ta * BM));
                    tma_load_3d(ssfa, &tmSFA, &full_bar[stage], 0, kt * 4, (int)ta);
                }
                if constexpr (!XQ) { // XQ: the activations are resident already
                    tma_load_2d(sb, &tmB, &full_bar[stage], kt * 128, 0);
                    tma_load_3d(ssfb, &tmSFB, &full_bar[stage], 0, kt * 4, 0);
                }
                ++issued;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            // every copy issued has landed before the CTA may exit
            int s = stage;
            uint32_t ph = phase;
            const int last = issued < C::kStages ? issued : C::kStages;
            for (int i = 0; i < last; ++i) {
                if (--s < 0) {
                    s = C::kStages - 1;
                    ph ^= 1;
                }
                if (!mbar_wait(&full_bar[s], ph, kWaitLimit))
                    set_timeout(p.status);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------- scale-factor feeders -----------------------
        const int q = warp & 3;
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        for (int kt = k0; kt < k1; ++kt) {
            if (!mbar_wait(&full_bar[stage], phase, kWaitLimit) ||
                !mbar_wait(&sf_empty[slot], sphase ^ 1, kWaitLimit)) {
                if (lane == 0)
                    set_timeout(p.status);
                break;
            }
            tc_fence_after();
            const uint32_t ssfa = smem_u32(smem + C::kOffSfa + stage * C::kSfaBytes);
            const uint32_t ssfb =
                smem_u32(smem + C::kOffSfb + (XQ ? kt - k0 : stage) * C::kSfbBytes);
            const uint32_t tslot =
                tmem + ((uint32_t)(q * 32) << 16) + C::kSfCol + slot * C::kSlotCols;
            uint32_t ra[16], rb[16];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const uint4 wa = lds128(ssfa + kb * 512 + lane * 16);
                const uint4 wb = lds128(ssfb + kb * 512 + lane * 16);
                ra[4 * kb] = wa.x;
                ra[4 * kb + 1] = wa.y;
                ra[4 * kb + 2] = wa.z;
                ra[4 * kb + 3] = wa.w;
                rb[4 * kb] = wb.x;
                rb[4 * kb + 1] = wb.y;
                rb[4 * kb + 2] = wb.z;
                rb[4 * kb + 3] = wb.w;
            }
            tmem_st_32x32b_x16(tslot, ra);
            tmem_st_32x32b_x16(tslot + 16, rb);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sf_full[slot]);
            if (++stage == C::kStages) {
                stage = 0;
                phase ^= 1;
            }
            if (++slot == C::kSfSlots) {
                slot = 0;
                sphase ^= 1;
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        bool ok = true;
        for (int kt = k0; kt < k1; ++kt) {
            if (!mbar_wait(&full_bar[stage], phase, kWaitLimit) ||
                !mbar_wait(&sf_full[slot], sphase, kWaitLimit)) {
                if (lane == 0)
                    set_timeout(p.status);
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t tsfa = tmem + C::kSfCol + slot * C::kSlotCols;
                const uint64_t adesc = smem_desc(smem_u32(smem + stage * C::kABytes), 16, 1024,
                                                 kLayoutSwizzle128B);
                const uint64_t bdesc =
                    smem_desc(smem_u32(smem + C::kOffB + (XQ ? kt - k0 : stage) * C::kBBytes), 16,
                              1024, kLayoutSwizzle128B);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
                    tc_mma_nvf4(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb),
                                C::kIdesc, tsfa + kb * 4, tsfa + 16 + kb * 4,
                                (kt > k0 || kb > 0) ? 1u : 0u);
                tc_commit(&empty_bar[stage]);
                tc_commit(&sf_empty[slot]);
            }
            __syncwarp();
            if (++stage == C::kStages) {
                stage = 0;
                phase ^= 1;
            }
            if (++slot == C::kSfSlots) {
                slot = 0;
                sphase ^= 1;
            }
        }
        if (lane == 0) {
            if (ok)
                tc_commit(acc_full);
            tc_commit(drain_bar); // every MMA issued completes before TMEM is freed
            if (!mbar_wait(drain_bar, 0, kWaitLimit))
                set_timeout(p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue (warps 2..5) ----------------------
        // partial accumulator -> own shared memory, [BN][128] fp32 (row m of the output
        // tile = accumulator column, 128 output columns n = TMEM lanes), over the drained
        // operand stages
        const int q = warp & 3;
        const int t = q * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        constexpr int NC = BN < 32 ? BN : 32;
        pdl_wait(); // global scales and y belong to the stream's earlier work
        alpha = __fmul_rn(XQ ? sg_x : *p.a_gs, *p.w_gs);
        const bool ok = mbar_wait(acc_full, 0, kWaitLimit);
        if (!ok && lane == 0)
            set_timeout(p.status);
        tc_fence_after();
        float *part = reinterpret_cast<float *>(smem);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += NC) {
            uint32_t v[NC];
            tmem_ld_cols<NC>(trow + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < NC; ++j)
                part[(c0 + j) * BM + t] = (ok && k1 > k0) ? __uint_as_float(v[j]) : 0.0f;
        }
    }

    __syncwarp();
    tc_fence_before();
    if (cs > 1)
        cluster_sync(); // every CTA of the cluster has staged its partial
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols); // the accumulator has been read
    }
    if (warp >= 2 && warp <= 5) {
        const int t = (warp & 3) * 32 + lane;
        switch (cs) {
        case 1: reduce_slice<BN, 1>(p, smem, 0, t, ta, alpha, &tmY); break;
        case 2: reduce_slice<BN, 2>(p, smem, rank, t, ta, alpha, &tmY); break;
        case 4: reduce_slice<BN, 4>(p, smem, rank, t, ta, alpha, &tmY); break;
        default: reduce_slice<BN, 8>(p, smem, rank, t, ta, alpha, &tmY); break;
        }
    } else if (cs > 1) {
        __syncwarp();
        cluster_arrive();
    }
    __syncwarp();
    if (cs > 1)
        cluster_wait(); // no CTA leaves while another may still read its partial
}

// Same threads and shared memory as nvfp4_gemm_smallm_kernel<BN> but no tensor memory. The
// occupancy calculator counts a CTA that allocates tensor memory as filling its SM, while two
// small-M CTAs (2 x 256 of the 512 columns) do run side by side; this kernel, never launched,
// gives the calculator's count of resident clusters for that shape.
template <int BN> __global__ void __launch_bounds__(kThreads, 2) smallm_occupancy_proxy(int *p)
{
    extern __shared__ uint8_t proxy_smem[];
    if (p)
        p[threadIdx.x] = proxy_smem[threadIdx.x];
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

// bf16 output Y [rows x cols], box 64 columns x 128 rows, 128B swizzle (TMA store).
bool make_out_map(CUtensorMap *m, void *base, int64_t rows, int64_t cols)
{
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {64u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output Y [M x N] (bf16 or fp32) of the small-M kernel, box 128 columns x box_rows rows, no
// swizzle: one CTA's staged slice of the output tile.
bool make_out_map_swap(CUtensorMap *m, void *base, int64_t rows, int64_t cols, int bf16,
                       int box_rows)
{
    const cuuint64_t esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * esz};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return encode_fn()(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                       2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_bn(const LinearPlan &pl, const uint8_t *a_codes, const uint8_t *a_sf,
                      const uint8_t *b_codes, const uint8_t *b_sf, int64_t K, GemmParams gp,
                      cudaStream_t s, nvfp4_status *st)
{
    using C = Cfg<BN>;
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmY;
    memset(&tmY, 0, sizeof(tmY));
    gp.tma_store = 0;
    if (BN == 256 && gp.splits == 1 && gp.out_bf16 && !gp.swap && gp.ldy % 8 == 0 &&
        (reinterpret_cast<uintptr_t>(gp.y) & 15u) == 0 && encode_fn() &&
        make_out_map(&tmY, gp.y, gp.rows_a, gp.rows_b))
        gp.tma_store = 1;
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
                                                                          tmSFB, tmY, gp);
    return cudaGetLastError();
}

// LR: lr_t (T' [M x lr_rank] bf16) and lr_u (U [N x lr_rank] bf16) feed the low-rank k-tiles.
template <bool QOUT, bool LR = false>
cudaError_t launch_pair(const uint8_t *a_codes, const uint8_t *a_sf, const uint8_t *w_codes,
                        const uint8_t *w_sf, int64_t M, int64_t N, int64_t K, GemmParams gp,
                        cudaStream_t s, nvfp4_status *st, const void *lr_t = nullptr,
                        const void *lr_u = nullptr, int lr_rank = 0)
{
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmY, tmT, tmU;
    std::memset(&tmY, 0, sizeof(tmY));
    std::memset(&tmT, 0, sizeof(tmT));
    std::memset(&tmU, 0, sizeof(tmU));
    if (!encode_fn() || !make_codes_map(&tmA, a_codes, M, K, 128) ||
        !make_codes_map(&tmB, w_codes, N, K, 128) || !make_sf_map(&tmSFA, a_sf, M, K, 1) ||
        !make_sf_map(&tmSFB, w_sf, N, K, 2) || (!QOUT && !make_out_map(&tmY, gp.y, M, N)) ||
        (LR && (!make_bf16_kmajor_map(&tmT, lr_t, M, lr_rank, 128) ||
                !make_bf16_kmajor_map(&tmU, lr_u, N, lr_rank, 128)))) {
        *st = NVFP4_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    gp.lr_kt = LR ? (lr_rank + 63) / 64 : 0;
    static std::once_flag flags[64];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t attr_err = cudaSuccess;
    std::call_once(flags[dev & 63], [&]() {
        attr_err = cudaFuncSetAttribute(nvfp4_gemm_pair_kernel<QOUT, LR>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Pair<QOUT>::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return attr_err;
    gp.tiles_a = (M + 255) / 256;
    gp.tiles_b = (N + 255) / 256;
    gp.units = gp.tiles_a * gp.tiles_b;
    int64_t clusters = num_sms() / 2;
    if (clusters > gp.units)
        clusters = gp.units;
    if (clusters < 1)
        clusters = 1;
    // programmatic dependent launch: barrier set-up, TMEM allocation and the cluster barrier
    // overlap the previous kernel's tail; the producer and the epilogue wait for it before
    // touching its outputs
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Pair<QOUT>::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, nvfp4_gemm_pair_kernel<QOUT, LR>, tmA, tmB, tmSFA, tmSFB, tmY,
                              tmT, tmU, gp);
}

template <int BN, bool XQ = false> cudaError_t smallm_set_smem_attr()
{
    static std::once_flag flags[64];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t e = cudaSuccess;
    std::call_once(flags[dev & 63], [&]() {
        e = cudaFuncSetAttribute(nvfp4_gemm_smallm_kernel<BN, XQ>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SmallCfg<BN, XQ>::L::kSmemBytes);
        if (e == cudaSuccess && !XQ)
            e = cudaFuncSetAttribute(smallm_occupancy_proxy<BN>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SmallCfg<BN>::L::kSmemBytes);
    });
    return e;
}

// Clusters of cs CTAs of the small-M kernel that can be resident at once on this device.
template <int BN> int smallm_max_clusters(int cs)
{
    if (smallm_set_smem_attr<BN>() != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(cs * 1024), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SmallCfg<BN>::L::kSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, smallm_occupancy_proxy<BN>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

constexpr int kMaxCsplit = 8; // portable cluster size

// Resident clusters per cluster size 1..8 for each small-M tile width, per device.
struct SmallOccupancy {
    int clusters[5][kMaxCsplit + 1];
};

const SmallOccupancy &small_occupancy()
{
    static std::once_flag flags[64];
    static SmallOccupancy occ[64];
    int dev = 0;
    cudaGetDevice(&dev);
    dev &= 63;
    std::call_once(flags[dev], [&]() {
        for (int cs = 1; cs <= kMaxCsplit; ++cs) {
            occ[dev].clusters[0][cs] = smallm_max_clusters<8>(cs);
            occ[dev].clusters[1][cs] = smallm_max_clusters<16>(cs);
            occ[dev].clusters[2][cs] = smallm_max_clusters<32>(cs);
            occ[dev].clusters[3][cs] = smallm_max_clusters<64>(cs);
            occ[dev].clusters[4][cs] = smallm_max_clusters<128>(cs);
        }
    });
    return occ[dev];
}

int bn_index(int bn) { return bn <= 8 ? 0 : bn <= 16 ? 1 : bn <= 32 ? 2 : bn <= 64 ? 3 : 4; }

template <int BN, bool XQ = false>
cudaError_t launch_smallm(const LinearPlan &pl, const uint8_t *w_codes, const uint8_t *w_sf,
                          const uint8_t *a_codes, const uint8_t *a_sf, int64_t K,
                          const SmallParams &sp, cudaStream_t s, nvfp4_status *st)
{
    using C = typename SmallCfg<BN, XQ>::L;
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmY;
    memset(&tmY, 0, sizeof(tmY));
    memset(&tmB, 0, sizeof(tmB));
    memset(&tmSFB, 0, sizeof(tmSFB));
    SmallParams spl = sp;
    spl.tma_store = 0;
    const int64_t esz = sp.out_bf16 ? 2 : 4;
    if ((sp.ldy * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(sp.y) & 15u) == 0 &&
        encode_fn() && make_out_map_swap(&tmY, sp.y, pl.rows_b, sp.ldy, sp.out_bf16, BN / pl.csplit))
        spl.tma_store = 1;
    if (!encode_fn() || !make_codes_map(&tmA, w_codes, pl.rows_a, K, BM) ||
        !make_sf_map(&tmSFA, w_sf, pl.rows_a, K, 1) ||
        (!XQ && (!make_codes_map(&tmB, a_codes, pl.rows_b, K, BN) ||
                 !make_sf_map(&tmSFB, a_sf, pl.rows_b, K, 1)))) {
        *st = NVFP4_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    cudaError_t e = smallm_set_smem_attr<BN, XQ>();
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(pl.tiles_a * pl.csplit), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    int na = 0;
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (pl.csplit > 1) {
        at[na].id = cudaLaunchAttributeClusterDimension;
        at[na].val.clusterDim.x = (unsigned)pl.csplit;
        at[na].val.clusterDim.y = 1;
        at[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = at;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, nvfp4_gemm_smallm_kernel<BN, XQ>, tmA, tmB, tmSFA, tmSFB,
                              tmY, spl);
}

} // namespace

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, unsigned flags)
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
    p.csplit = 0;
    const int64_t tiles = p.tiles_a * p.tiles_b;
    if (p.swap_ab) {
        // One wave of clusters: the largest K split (8, 4 or 2, at most the k-tiles; a power
        // of two so that it divides the tile width) whose clusters of one tile each are all
        // resident at once; shapes with more tiles than one wave of single CTAs go to the
        // persistent kernel.
        // The grid stays within 4/3 of the SM count: a few SMs run two CTAs, the rest keep a
        // slot free for the next kernel's CTAs (they start streaming resident weights there).
        // Measured on 8 x {6144, 12288, 18944} x 4096: more CTAs only lengthen the tail.
        (void)flags;
        const SmallOccupancy &occ = small_occupancy();
        const int bi = bn_index(p.bn);
        const int64_t max_ctas = (int64_t)num_sms() * 4 / 3;
        for (int cs = kMaxCsplit; cs >= 1; cs /= 2) {
            if (cs <= p.kt && tiles <= occ.clusters[bi][cs] && (cs == 1 || tiles * cs <= max_ctas)) {
                p.csplit = cs;
                break;
            }
        }
        if (p.csplit > 0) {
            p.ws_bytes = 0;
            return p;
        }
    }
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

cudaError_t launch_linear_nvfp4_out(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gs,
                                    const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                                    int64_t M, int64_t N, int64_t K, int act,
                                    const float *static_amax, uint8_t *y_codes, uint8_t *y_sf,
                                    float *y_gs, cudaStream_t s, nvfp4_status *st)
{
    GemmParams gp{};
    gp.rows_a = M;
    gp.rows_b = N;
    gp.kt_total = (int)((K + 255) / 256);
    gp.kt_per_split = gp.kt_total;
    gp.splits = 1;
    gp.a_gs = a_gs;
    gp.w_gs = w_gs;
    gp.ldy = N;
    gp.status = device_status_ptr();
    gp.q_codes = y_codes;
    gp.q_sf = y_sf;
    gp.q_gs = y_gs;
    gp.q_amax = static_amax;
    gp.act = act;
    gp.q_apb = (int)((N / 16 + 3) / 4);
    gp.q_rows_pad = (M + 127) / 128 * 128;
    return launch_pair<true>(a_codes, a_sf, w_codes, w_sf, M, N, K, gp, s, st);
}

cudaError_t launch_linear(const LinearPlan &pl, const uint8_t *a_codes, const uint8_t *a_sf,
                          const float *a_gs, const uint8_t *w_codes, const uint8_t *w_sf,
                          const float *w_gs, int64_t M, int64_t N, int64_t K, int out_bf16,
                          void *y, void *ws, unsigned flags, cudaStream_t s, nvfp4_status *st)
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
    if (pl.csplit > 0) {
        SmallParams sp{};
        sp.rows_a = pl.rows_a;
        sp.rows_b = pl.rows_b;
        sp.kt_total = pl.kt;
        sp.csplit = pl.csplit;
        sp.a_gs = a_gs;
        sp.w_gs = w_gs;
        sp.y = y;
        sp.ldy = N;
        sp.out_bf16 = out_bf16;
        sp.resident_w = (flags & NVFP4_LINEAR_RESIDENT_WEIGHTS) ? 1 : 0;
        sp.status = device_status_ptr();
        switch (pl.bn) {
        case 8: return launch_smallm<8>(pl, ca, sa, cb, sb, K, sp, s, st);
        case 16: return launch_smallm<16>(pl, ca, sa, cb, sb, K, sp, s, st);
        case 32: return launch_smallm<32>(pl, ca, sa, cb, sb, K, sp, s, st);
        case 64: return launch_smallm<64>(pl, ca, sa, cb, sb, K, sp, s, st);
        default: return launch_smallm<128>(pl, ca, sa, cb, sb, K, sp, s, st);
        }
    }
    if (!pl.swap_ab && pl.splits == 1 && out_bf16 && N % 8 == 0 &&
        (reinterpret_cast<uintptr_t>(y) & 15u) == 0 && kUsePairKernel)
        return launch_pair<false>(a_codes, a_sf, w_codes, w_sf, M, N, K, gp, s, st);
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

// Fused dynamic-activation linear (M <= 16): the small-M plan with a cluster split whose
// per-CTA k-range holds at most kXqMaxKt k-tiles (the resident activation tiles). Returns
// false when the shape does not fit that. Above M = 16 the in-kernel quantize (every cluster
// reads the whole activation tensor for its amax) costs more than a separate quantize: on
// B200, N12288 K4096, fused vs quantize + linear: M16 14.9 vs 17.5 us, M24 18.5 vs 17.9 us.
bool plan_linear_xq(int64_t M, int64_t N, int64_t K, LinearPlan *out)
{
    if (M < 1 || M > 16 || N < 1 || K < 32)
        return false;
    LinearPlan p = plan_linear(M, N, K, 0);
    if (!p.swap_ab || p.bn > 32)
        return false;
    const SmallOccupancy &occ = small_occupancy();
    const int bi = bn_index(p.bn);
    const int64_t tiles = p.tiles_a;
    const int64_t max_ctas = (int64_t)num_sms() * 4 / 3;
    int csplit = 0;
    for (int cs = kMaxCsplit; cs >= 1; cs /= 2) {
        const bool fits = cs <= p.kt && tiles <= occ.clusters[bi][cs] &&
                          (cs == 1 || tiles * cs <= max_ctas) &&
                          (p.kt + cs - 1) / cs <= kXqMaxKt;
        if (fits) {
            csplit = cs;
            break;
        }
    }
    if (csplit == 0) { // the k-range would not stay resident: the largest resident split
        for (int cs = kMaxCsplit; cs >= 1; cs /= 2)
            if (cs <= p.kt && tiles <= occ.clusters[bi][cs] &&
                (p.kt + cs - 1) / cs <= kXqMaxKt) {
                csplit = cs;
                break;
            }
    }
    if (csplit == 0)
        return false;
    p.csplit = csplit;
    p.ws_bytes = 0;
    *out = p;
    return true;
}

// Linear layer with a BF16 low-rank branch: T' = bf16(x . D^T * RN(1 / alpha)) into t_ws (the down
// kernel), then the pair GEMM with the low-rank k-tiles appended to every tile. bf16 output.
cudaError_t launch_linear_lowrank(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gs,
                                  const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                                  const void *x, const void *lr_down, const void *lr_up,
                                  int64_t M, int64_t N, int64_t K, int rank, void *y, void *t_ws,
                                  cudaStream_t s, nvfp4_status *st)
{
    cudaError_t e = launch_lowrank_down(x, lr_down, M, K, rank, a_gs, w_gs, t_ws, s, st);
    if (e != cudaSuccess || *st != NVFP4_OK)
        return e;
    GemmParams gp{};
    gp.rows_a = M;
    gp.rows_b = N;
    gp.kt_total = (int)((K + 255) / 256);
    gp.kt_per_split = gp.kt_total;
    gp.splits = 1;
    gp.a_gs = a_gs;
    gp.w_gs = w_gs;
    gp.y = y;
    gp.ldy = N;
    gp.out_bf16 = 1;
    gp.status = device_status_ptr();
    return launch_pair<false, true>(a_codes, a_sf, w_codes, w_sf, M, N, K, gp, s, st, t_ws, lr_up,
                                    rank);
}

cudaError_t launch_linear_xq(const LinearPlan &pl, const void *x, int x_bf16,
                             const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                             int64_t M, int64_t N, int64_t K, int out_bf16, void *y,
                             float *x_gs_out, unsigned flags, cudaStream_t s, nvfp4_status *st)
{
    SmallParams sp{};
    sp.rows_a = pl.rows_a;
    sp.rows_b = pl.rows_b;
    sp.kt_total = pl.kt;
    sp.csplit = pl.csplit;
    sp.a_gs = nullptr;
    sp.w_gs = w_gs;
    sp.y = y;
    sp.ldy = N;
    sp.out_bf16 = out_bf16;
    sp.resident_w = (flags & NVFP4_LINEAR_RESIDENT_WEIGHTS) ? 1 : 0;
    sp.status = device_status_ptr();
    sp.x = x;
    sp.x_bf16 = x_bf16;
    sp.K = K;
    sp.x_gs_out = x_gs_out;
    (void)M;
    switch (pl.bn) {
    case 8: return launch_smallm<8, true>(pl, w_codes, w_sf, nullptr, nullptr, K, sp, s, st);
    case 16: return launch_smallm<16, true>(pl, w_codes, w_sf, nullptr, nullptr, K, sp, s, st);
    default: return launch_smallm<32, true>(pl, w_codes, w_sf, nullptr, nullptr, K, sp, s, st);
    }
}

// ---------------------------------------------------------------------------------------
// Allocation-free entry point
// ---------------------------------------------------------------------------------------

namespace {

// Split-K partial sums of nvfp4_linear_noalloc live here instead of in a caller-supplied
// workspace. Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20; // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kNoAllocMaxDevices]; // null until an address was resolved on that device

// Device address of the scratch array on the current device. In host code the array's name
// only stands for the symbol; the address kernels may use comes from cudaGetSymbolAddress,
// resolved with that device current. Only a successful lookup is kept: a failed one (for
// example a first call made while the stream is being captured) returns its error and the
// next call tries again.
cudaError_t noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

} // namespace

} // namespace nvfp4

extern "C" nvfp4_status nvfp4_linear_noalloc(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                             const float *a_gs, const uint8_t *w_codes,
                                             const uint8_t *w_scales_swz, const float *w_gs,
                                             int64_t M, int64_t N, int64_t K,
                                             nvfp4_dtype out_dt, void *y, cudaStream_t stream)
{
    using namespace nvfp4;
    size_t need = 0;
    if (M > 0 && N > 0 && K > 0 && K % 32 == 0 && M < ((int64_t)1 << 31) &&
        N < ((int64_t)1 << 31) && K < ((int64_t)1 << 31))
        need = plan_linear(M, N, K).ws_bytes;
    if (need > kNoAllocScratchBytes)
        return NVFP4_ERR_WORKSPACE; // this shape's split-K partials exceed the 4 MiB scratch
    void *scratch = nullptr;
    if (need > 0 && noalloc_scratch(&scratch) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return nvfp4_linear(a_codes, a_scales_swz, a_gs, w_codes, w_scales_swz, w_gs, M, N, K,
                        out_dt, y, scratch, scratch ? kNoAllocScratchBytes : 0, stream);
}
