// lowrank_sm100.cu -- down projection of a linear layer's BF16 low-rank branch on sm_100a.
//
// "Qwen Image 2.1: INT4 + FP4", section "What I quantized": the transformer's linear layers run
// in native FP4 on Blackwell next to BF16 rank-128 branches, Y = FP4 product + (x . D^T) . U^T
// with D [r x K] and U [N x r]. This file computes the branch's intermediate T = x . D^T from
// the layer's bf16 input on the tensor cores (tcgen05 kind::f16, fp32 accumulation) and stores
// it as bf16 of T * RN(1 / alpha), alpha = sgA * sgW (1 when that product is 0): the FP4 GEMM then adds
// T . U^T into its own accumulator, which its epilogue multiplies by alpha (gemm_sm100.cu,
// nvfp4_gemm_pair_kernel with the low-rank k-tiles).
//
// Shape of the work: M x r outputs (r <= 256) over K = 3072 is little arithmetic next to the
// bytes of x, so the kernel is HBM-bound on x. Each 128-row band of x is split along K over a
// thread-block cluster of up to 4 CTAs (128 CTAs for 4096 rows, one per SM), each streaming
// its K range of x and D through a 4-stage TMA ring into one M128 x N=r MMA accumulator in
// TMEM. The partial accumulators meet in shared memory: every CTA stages its partial, and
// after a cluster barrier each CTA sums its share of the band's rows over the cluster's
// partials in rank order (deterministic), multiplies by 1 / alpha, rounds to bf16 and stores.
// The other CTAs' rows of that share arrive by bulk copies that their senders push into this
// CTA's shared memory (remote loads of the same 48 KB a CTA took 3.4 us more, measured).
#include <cuda.h>
#include <cstring>
#include <mutex>

#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

// warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 epilogue; all 8 warps reduce the
// cluster's partials
constexpr int kDnThreads = 256;
// K split (CTAs per cluster, a power of two <= 8) and the most TMA ring stages (as many as the
// shared memory holds, up to this). Measured on M4096 K3072 r128: a split of 4 with one CTA per
// SM beats 8 with two CTAs per SM (3 stages each) and 8 with 4 stages; the loads are
// latency-bound, so the deepest ring that fits is taken.
#ifndef NVFP4_DN_SPLIT
#define NVFP4_DN_SPLIT 4
#endif
#ifndef NVFP4_DN_STAGES
#define NVFP4_DN_STAGES 6
#endif
constexpr int kDnMaxStages = NVFP4_DN_STAGES;
constexpr int kDnMaxSplit = NVFP4_DN_SPLIT;
constexpr int kDnSmemMax = 232448; // per-CTA shared memory limit
constexpr int kDnABytes = 128 * 128; // 128 rows of x x 64 bf16 (one 128-byte swizzle row)
constexpr uint32_t kDnWaitLimit = 1u << 20;

struct DownParams {
    int64_t M;
    int r;        // rank: multiple of 16, 16..256
    int stages;   // TMA ring depth (3 .. kDnMaxStages; the fp32 partial fits in 3 or more)
    int kt_total; // 64-wide k-tiles of K
    int push;     // 1: the partials' rows reach their summing CTA by pushed bulk copies into an
                  // inbox after the partial (dn_push_fits); 0: by remote loads
    const float *a_gs, *w_gs;
    __nv_bfloat16 *t; // [M x r], row stride r
    int *status;
};

__host__ __device__ constexpr int dn_stage_bytes(int r) { return kDnABytes + r * 128; }
__host__ __device__ constexpr uint32_t dn_tmem_cols(int r)
{
    return r <= 32 ? 32u : r <= 64 ? 64u : r <= 128 ? 128u : 256u;
}
constexpr int dn_stages(int r)
{
    return (kDnSmemMax - 256) / dn_stage_bytes(r) < kDnMaxStages
               ? (kDnSmemMax - 256) / dn_stage_bytes(r)
               : kDnMaxStages;
}
constexpr int dn_smem_bytes(int r) { return dn_stages(r) * dn_stage_bytes(r) + 256; }
// fp32 partial rows of r + 4 floats (the pad spreads a warp's row-strided stores over the banks)
__host__ __device__ constexpr uint32_t dn_row_bytes(int r) { return (uint32_t)(r + 4) * 4u; }
// the partial (128 rows) and an inbox of another 128 rows fit in the drained stage buffers
constexpr bool dn_push_fits(int r)
{
    return 256u * dn_row_bytes(r) <= (uint32_t)(dn_stages(r) * dn_stage_bytes(r));
}
static_assert(dn_push_fits(128) && dn_push_fits(192), "push reduce for the usual ranks");
static_assert(dn_stages(256) >= 3 && dn_stages(16) >= 3, "ring depth");
constexpr int dn_smem_max()
{
    int m = 0;
    for (int r = 16; r <= 256; r += 16)
        m = dn_smem_bytes(r) > m ? dn_smem_bytes(r) : m;
    return m;
}
static_assert(dn_smem_max() <= kDnSmemMax, "shared memory");

__device__ __forceinline__ void dn_timeout(int *status)
{
    atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
}

// D(tmem) (+)= A(smem) x B(smem)^T, bf16 x bf16 -> fp32, one CTA.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

__device__ __forceinline__ float4 ld_shared_cluster_f32x4(uint32_t cluster_addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}

// Bulk copy of `bytes` from this CTA's shared memory to a cluster shared-memory address
// (dst, mbar: mapa addresses in the receiving CTA); completes as bytes on the receiver's
// mbarrier; exactly one destination CTA.
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst, uint32_t src, uint32_t bytes,
                                                     uint32_t mbar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes "
                 "[%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// grid (S, ceil(M / 128)), cluster (S, 1, 1): CTA (rank, band) takes k-tiles
// [kt_total * rank / S, kt_total * (rank + 1) / S) of rows [128 band, 128 band + 128).
__global__ void __launch_bounds__(kDnThreads, 1)
    lowrank_down_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmD, const DownParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    // programmatic dependent launch: the set-up below overlaps the previous kernel's tail; the
    // producer (x) and the reduce (the global scales, T's earlier readers) wait for it
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = p.r;
    const int stage_bytes = dn_stage_bytes(r);
    const uint32_t S = gridDim.x;
    const uint32_t rank = cluster_ctarank();
    const int64_t band = blockIdx.y;
    const int nst = p.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + nst * stage_bytes);
    uint64_t *empty = full + kDnMaxStages;
    uint64_t *acc_full = empty + kDnMaxStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    uint64_t *inbox_full = acc_full + 2; // push reduce: the other CTAs' rows have arrived
    const bool aligned = (smem_u32(smem) & 1023u) == 0; // uniform over the cluster
    const int kt0 = (int)((int64_t)p.kt_total * rank / S);
    const int nk = (int)((int64_t)p.kt_total * (rank + 1) / S) - kt0; // >= 1 unless K == 0
    const uint32_t tcols = dn_tmem_cols(r);

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(inbox_full, 1);
        fence_barrier_init();
        if (!aligned)
            atomicExch(p.status, (int)NVFP4_ERR_CUDA);
    }
    if (warp == 1 && aligned) {
        tmem_alloc(tmem_slot, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = aligned ? *tmem_slot : 0u;

    if (!aligned) {
        // nothing runs; the CTAs still meet at both cluster barriers below
    } else if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmD);
            pdl_wait();
            for (int i = 0; i < nk; ++i) {
                const int s = i % nst;
                const uint32_t ph = (uint32_t)(i / nst) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, kDnWaitLimit)) {
                    dn_timeout(p.status);
                    break;
                }
                mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
                tma_load_2d(smem + s * stage_bytes, &tmX, &full[s], (kt0 + i) * 64,
                            (int)(band * 128));
                tma_load_2d(smem + s * stage_bytes + kDnABytes, &tmD, &full[s], (kt0 + i) * 64, 0);
            }
        }
    } else if (warp == 1) {
        // kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9 and
        // 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24 (M = 128)
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(r >> 3) << 17) |
                               ((uint32_t)(128 >> 4) << 24);
        for (int i = 0; i < nk; ++i) {
            const int s = i % nst;
            const uint32_t ph = (uint32_t)(i / nst) & 1u;
            if (!mbar_wait(&full[s], ph, kDnWaitLimit)) {
                if (lane == 0)
                    dn_timeout(p.status);
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sa = smem_u32(smem + s * stage_bytes);
                const uint64_t adesc = smem_desc(sa, 16, 1024, kLayoutSwizzle128B);
                const uint64_t bdesc = smem_desc(sa + kDnABytes, 16, 1024, kLayoutSwizzle128B);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) // 16 bf16 = 32 bytes per MMA along K
                    tc_mma_bf16(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb), idesc,
                                (i > 0 || kb > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            __syncwarp();
        }
        if (lane == 0)
            tc_commit(acc_full); // also after a timeout, once the issued MMAs complete
        __syncwarp();
    } else if (warp < 6) {
        // epilogue: this warp's 32 TMEM lanes = rows q*32 .. q*32+31 of the band
        const int q = warp & 3;
        const int row = q * 32 + lane;
        // partial [128 x (r + 4)] fp32 over the drained stage buffers; the 16-byte pad
        // spreads a warp's row-strided stores over distinct banks
        const uint32_t prow = smem_u32(smem) + (uint32_t)(row * (r + 4) * 4);
        if (!mbar_wait(acc_full, 0, kDnWaitLimit)) {
            if (lane == 0)
                dn_timeout(p.status);
        } else if (nk == 0) { // K == 0: no MMA wrote the accumulator
            for (int c = 0; c < r; c += 4)
                sts128(prow + (uint32_t)(c * 4), 0u, 0u, 0u, 0u);
        } else {
            tc_fence_after();
            fence_proxy_async_smem();
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
            int c = 0;
            for (; c + 32 <= r; c += 32) { // two 16-column loads per wait
                uint32_t v[32];
                tmem_ld_32x32b_x16(trow + (uint32_t)c, v);
                tmem_ld_32x32b_x16(trow + (uint32_t)c + 16u, v + 16);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    sts128(prow + (uint32_t)((c + j) * 4), v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
            if (c < r) { // r % 32 == 16
                uint32_t v[16];
                tmem_ld_32x32b_x16(trow + (uint32_t)c, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    sts128(prow + (uint32_t)((c + j) * 4), v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
        fence_proxy_async_smem(); // the partial's rows, before bulk copies read them
    }
    const int rows_per = 128 / (int)S;
    const uint32_t chunk = (uint32_t)rows_per * dn_row_bytes(r); // one CTA's share of a partial
    if (threadIdx.x == 0 && aligned && p.push && S > 1)
        mbar_arrive_expect_tx(inbox_full, (S - 1) * chunk); // armed before any copy can land
    tc_fence_before();
    __syncwarp();
    cluster_sync(); // every partial of the cluster is in shared memory
    pdl_launch_dependents(); // the GEMM may set up while the partials are reduced

    if (aligned) {
        pdl_wait();
        float alpha = __fmul_rn(*p.a_gs, *p.w_gs);
        if (alpha == 0.0f)
            alpha = 1.0f; // the FP4 product is zero then; the GEMM scales by 1 as well
        const float ralpha = __frcp_rn(alpha);
        const int v8 = r / 8;
        const int nitems = rows_per * v8;
        const uint32_t base = smem_u32(smem);
        const uint32_t rb = dn_row_bytes(r);
        if (p.push) {
            // rows [rows_per d, rows_per (d + 1)) of this CTA's partial go to CTA d's inbox,
            // slot `rank`; this CTA's own share stays where it is
            const uint32_t inbox = base + 128u * rb;
            if (threadIdx.x == 0)
                for (uint32_t d = 0; d < S; ++d)
                    if (d != rank)
                        bulk_copy_to_cluster(mapa_shared(inbox + rank * chunk, d),
                                             base + d * chunk, chunk,
                                             mapa_shared(smem_u32(inbox_full), d));
            if (S > 1 && !mbar_wait_cluster(inbox_full, 0, kDnWaitLimit)) {
                if (threadIdx.x == 0)
                    dn_timeout(p.status);
            } else {
                for (int idx = threadIdx.x; idx < nitems; idx += kDnThreads) {
                    const int lr = idx / v8;
                    const int c = (idx % v8) * 8;
                    const int64_t m = band * 128 + (int64_t)rank * rows_per + lr;
                    if (m >= p.M)
                        continue;
                    float acc[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        acc[j] = 0.0f;
#pragma unroll
                    for (int s = 0; s < kDnMaxSplit; ++s) // rank order: the same sum every run
                        if (s < (int)S) {
                            const uint32_t a =
                                ((uint32_t)s == rank ? base + rank * chunk : inbox + s * chunk) +
                                (uint32_t)lr * rb + (uint32_t)c * 4u;
                            const uint4 u0 = lds128(a), u1 = lds128(a + 16);
                            acc[0] += __uint_as_float(u0.x);
                            acc[1] += __uint_as_float(u0.y);
                            acc[2] += __uint_as_float(u0.z);
                            acc[3] += __uint_as_float(u0.w);
                            acc[4] += __uint_as_float(u1.x);
                            acc[5] += __uint_as_float(u1.y);
                            acc[6] += __uint_as_float(u1.z);
                            acc[7] += __uint_as_float(u1.w);
                        }
                    uint4 o;
                    o.x = bf16x2_bits(__fmul_rn(acc[0], ralpha), __fmul_rn(acc[1], ralpha));
                    o.y = bf16x2_bits(__fmul_rn(acc[2], ralpha), __fmul_rn(acc[3], ralpha));
                    o.z = bf16x2_bits(__fmul_rn(acc[4], ralpha), __fmul_rn(acc[5], ralpha));
                    o.w = bf16x2_bits(__fmul_rn(acc[6], ralpha), __fmul_rn(acc[7], ralpha));
                    *reinterpret_cast<uint4 *>(p.t + m * r + c) = o;
                }
            }
        } else {
        // two items a thread per pass, every rank's loads of both in flight before the sums
        for (int i0 = threadIdx.x; i0 < nitems; i0 += 2 * kDnThreads) {
            float4 lo[2][kDnMaxSplit], hi[2][kDnMaxSplit];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int idx = i0 + h * kDnThreads;
                if (idx >= nitems)
                    break;
                const int lr = (int)rank * rows_per + idx / v8;
                const uint32_t off =
                    base + (uint32_t)((lr * (r + 4) + (idx % v8) * 8) * 4);
#pragma unroll
                for (int s = 0; s < kDnMaxSplit; ++s)
                    if (s < (int)S) {
                        lo[h][s] = ld_shared_cluster_f32x4(mapa_shared(off, (uint32_t)s));
                        hi[h][s] = ld_shared_cluster_f32x4(mapa_shared(off + 16, (uint32_t)s));
                    }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int idx = i0 + h * kDnThreads;
                if (idx >= nitems)
                    break;
                const int lr = (int)rank * rows_per + idx / v8;
                const int c = (idx % v8) * 8;
                const int64_t m = band * 128 + lr;
                if (m >= p.M)
                    continue;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    acc[j] = 0.0f;
#pragma unroll
                for (int s = 0; s < kDnMaxSplit; ++s) // rank order: the same sum on every run
                    if (s < (int)S) {
                        acc[0] += lo[h][s].x;
                        acc[1] += lo[h][s].y;
                        acc[2] += lo[h][s].z;
                        acc[3] += lo[h][s].w;
                        acc[4] += hi[h][s].x;
                        acc[5] += hi[h][s].y;
                        acc[6] += hi[h][s].z;
                        acc[7] += hi[h][s].w;
                    }
                uint4 o;
                o.x = bf16x2_bits(__fmul_rn(acc[0], ralpha), __fmul_rn(acc[1], ralpha));
                o.y = bf16x2_bits(__fmul_rn(acc[2], ralpha), __fmul_rn(acc[3], ralpha));
                o.z = bf16x2_bits(__fmul_rn(acc[4], ralpha), __fmul_rn(acc[5], ralpha));
                o.w = bf16x2_bits(__fmul_rn(acc[6], ralpha), __fmul_rn(acc[7], ralpha));
                *reinterpret_cast<uint4 *>(p.t + m * r + c) = o;
            }
        }
        }
    }
    __syncwarp();
    cluster_sync(); // no CTA leaves while another may still read its partial
    if (warp == 1 && aligned) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn dn_encode_fn()
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

} // namespace

// bf16 [rows x cols] row-major, box 64 columns x box_rows rows, 128B swizzle; columns and rows
// past the matrix read as zero.
bool make_bf16_kmajor_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                          int box_rows)
{
    if (!dn_encode_fn())
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return dn_encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_lowrank_down(const void *x, const void *d, int64_t M, int64_t K, int r,
                                const float *a_gs, const float *w_gs, void *t, cudaStream_t s,
                                nvfp4_status *st)
{
    if (M == 0)
        return cudaSuccess;
    CUtensorMap tmX, tmD;
    if (!make_bf16_kmajor_map(&tmX, x, M, K, 128) || !make_bf16_kmajor_map(&tmD, d, r, K, r)) {
        *st = NVFP4_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    const int smem = dn_smem_bytes(r);
    static std::once_flag flags[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(flags[dev & 63], [&]() {
        attr_err[dev & 63] = cudaFuncSetAttribute(lowrank_down_kernel,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  dn_smem_max());
    });
    if (attr_err[dev & 63] != cudaSuccess)
        return attr_err[dev & 63];
    DownParams p{};
    p.M = M;
    p.r = r;
    p.stages = dn_stages(r);
    p.kt_total = (int)((K + 63) / 64);
    p.push = dn_push_fits(r) ? 1 : 0;
    p.a_gs = a_gs;
    p.w_gs = w_gs;
    p.t = reinterpret_cast<__nv_bfloat16 *>(t);
    p.status = device_status_ptr();
    // the largest power-of-two split (<= 8, so a band's 128 rows divide evenly) that leaves
    // every CTA at least one k-tile
    int S = 1;
    while (S * 2 <= kDnMaxSplit && S * 2 <= p.kt_total)
        S *= 2;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)S, (unsigned)((M + 127) / 128), 1);
    cfg.blockDim = dim3(kDnThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)S;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, lowrank_down_kernel, tmX, tmD, p);
}

} // namespace nvfp4
