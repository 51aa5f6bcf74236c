// quantize.cu -- NVFP4 quantization of fp32 / bf16 / FP8-E4M3 tensors on sm_100a.
//
// Format and decode rule: "Qwen-Image NVFP4 on a 16 GB Ada GPU", section "What NVFP4 is and
// how it differs from NF4" (E2M1 codes, one FP8 scale per 16 values, one FP32 global scale)
// and the figure "First NVFP4 block, as stored in the file" (low nibble first,
// weight = E2M1 x block scale x global scale). Dynamic per-tensor amax for activations:
// "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details". FP8 source (double
// quantization): "Qwen-Rapid-AIO FP8 -> NVFP4", "1. Double Quantization".
//
// Tensors of 16 MB up to what the CTAs' shared memory holds (148 x 192 KB) take one fused
// single-pass kernel (fused_quantize_kernel, below); larger ones take one streamed launch that
// reads the tensor twice through a shared-memory ring, amax then encode
// (stream_quantize_kernel); two tensors of a batch, the larger of the fused size and the
// smaller up to what the threads' registers hold, take one fused launch together
// (fused_pair_quantize_kernel). Tensors below 16 MB, and batches the pair launch does not fit
// (amax_group_kernel / encode_group_kernel, one launch of each for all the batch's tensors),
// take two kernels, both HBM-bound, chained by programmatic dependent launch:
//   amax_kernel   (dynamic amax only) -- one CTA per SM streams a contiguous byte range of
//                 the tensor (whole 16-byte vectors) through a 4 x 32 KB shared-memory ring of
//                 1-D bulk copies and reduces max |x| with native packed max (exact,
//                 order-free); one partial per CTA, no atomics, nothing to zero.
//   encode_kernel -- one CTA per SM owns a contiguous range of rows, taken from its end
//                 backwards (the part the amax pass left in L2 first); each warp takes a
//                 64-block run of one row (1024 values, fully coalesced), two 16-value blocks
//                 per lane. It loads its first items before griddepcontrol.wait, so the loads
//                 overlap the amax kernel's tail, reduces the partial maxima to the global
//                 scale, and fills a 128-entry table of 1 / (E4M3(c) * sg). Per block: block
//                 amax, E4M3 scale, E2M1 codes by the hardware cvt, a 16-byte code store (a warp
//                 writes 512 contiguous bytes) and 16-bit stores of the swizzled and / or linear
//                 scales; atom padding is zeroed.
// The FP8 E4M3 tensorwise quantizer at the end of the file follows the same plan (a single
// pass for 16 MB and up, amax + encode otherwise).
// Code-deciding arithmetic is IEEE fp32 round-to-nearest in a fixed order (__fdiv_rn,
// __fmul_rn, __frcp_rn): sg = amax / 2688, sb = E4M3(bmax / (sg * 6)),
// code = E2M1(x * (1 / (sb * sg))).
#include <mutex>

#include "encode_lean.cuh"
#include "grid_exchange.cuh"
#include "nvfp4_internal.cuh"
#include "nvfp4_encode.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kAmaxThreads = 1024;  // amax: one CTA per SM streaming its byte range
constexpr int kChunk = 32 * 1024;   // amax ring: 4 x 32 KB bulk copies in flight per SM
constexpr int kRing = 4;
constexpr int kFusedThreads = 1024;    // fused quantizer: one CTA per SM
constexpr int kFusedChunk = 32 * 1024;  // fused quantizer: bulk-copy size
constexpr int kFusedMaxChunks = 6;
constexpr int kFusedCap = kFusedChunk * kFusedMaxChunks; // tensor bytes per CTA (192 KB)
constexpr int kMaxQuantJobs = NVFP4_MAX_QUANT_JOBS; // tensors per batched quantize
// encode: 24 warps, two 16-value blocks per lane per item (up to 80 registers a thread; at
// 1024 threads the 64-register cap spills; measured 768 >= 1024 and 512 on 0.1-100 MB)
constexpr int kEncThreads = 768;
// The fused kernel runs tensors from kFusedMinBytes up to its shared-memory capacity. Below,
// its grid-wide barrier and one-CTA-per-SM launch cost more than the second kernel and the
// second read (from L2) save: measured on B200, bf16 / fp32 / fp8 from 0.1 to 25 MB, the
// fused kernel is ahead from about 12-16 MB (fp32 12.6 MB: 10.4 vs 11.5 us; bf16 25 MB:
// 14.1 vs 14.9 us) and behind below (bf16 6.3 MB: 8.6 vs 7.3 us).
constexpr int64_t kFusedMinBytes = (int64_t)16 << 20;
constexpr uint32_t kSpinLimit = 1u << 24;
// poll rounds of the fused kernels' grid exchange (each an L2 round trip, ~0.5-1 us): about
// a second before a missing CTA is reported as a timeout
constexpr uint32_t kExchangeLimit = 1u << 21;

template <int SRC> struct Src;

// Maxima of |x| are folded into a 32-bit container per source type, with native max
// instructions (exact, order-free): fp32 -> the float max itself; bf16 -> a bf16x2 pair of
// magnitudes (packed bf16 max, two values an instruction); fp8 -> an f16x2 pair of |e|
// (E4M3 widens to f16 exactly; packed f16 max). mag_to_f32 gives the maximum as fp32 (fp8:
// of |e|, before the fp8 scale).
__device__ __forceinline__ uint32_t hmax2_bf16(uint32_t a, uint32_t b)
{
    __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162 *>(&a),
                               *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t hmax2_f16(uint32_t a, uint32_t b)
{
    __half2 r = __hmax2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

// two E4M3 bytes -> f16x2 of their magnitudes (exact)
__device__ __forceinline__ uint32_t e4m3x2_abs_to_f16x2(uint32_t b2)
{
    uint32_t h;
    const uint16_t in = (uint16_t)(b2 & 0x7F7Fu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
    return h;
}

template <> struct Src<kSrcF32> {
    static constexpr int kBytes = 4;
    __device__ static uint32_t vec_magmax(uint4 v)
    {
        return __float_as_uint(fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                                     fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
    }
    __device__ static uint32_t fold(uint32_t a, uint32_t b) { return max(a, b); }
    __device__ static float mag_to_f32(uint32_t m) { return __uint_as_float(m); }
};

template <> struct Src<kSrcBF16> {
    static constexpr int kBytes = 2;
    __device__ static uint32_t vec_magmax(uint4 v)
    {
        const uint32_t k = 0x7FFF7FFFu;
        return hmax2_bf16(hmax2_bf16(v.x & k, v.y & k), hmax2_bf16(v.z & k, v.w & k));
    }
    __device__ static uint32_t fold(uint32_t a, uint32_t b) { return hmax2_bf16(a, b); }
    __device__ static float mag_to_f32(uint32_t m)
    {
        return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    }
};

template <> struct Src<kSrcE4M3> {
    static constexpr int kBytes = 1;
    __device__ static uint32_t vec_magmax(uint4 v)
    {
        const uint32_t a = hmax2_f16(e4m3x2_abs_to_f16x2(v.x), e4m3x2_abs_to_f16x2(v.x >> 16));
        const uint32_t b = hmax2_f16(e4m3x2_abs_to_f16x2(v.y), e4m3x2_abs_to_f16x2(v.y >> 16));
        const uint32_t c = hmax2_f16(e4m3x2_abs_to_f16x2(v.z), e4m3x2_abs_to_f16x2(v.z >> 16));
        const uint32_t d = hmax2_f16(e4m3x2_abs_to_f16x2(v.w), e4m3x2_abs_to_f16x2(v.w >> 16));
        return hmax2_f16(hmax2_f16(a, b), hmax2_f16(c, d));
    }
    __device__ static uint32_t fold(uint32_t a, uint32_t b) { return hmax2_f16(a, b); }
    __device__ static float mag_to_f32(uint32_t m) // |e4m3| (before the fp8 scale)
    {
        const __half2 h = *reinterpret_cast<const __half2 *>(&m);
        return fmaxf(__low2float(h), __high2float(h));
    }
};


// Fold a magnitude accumulator (per source type) into another.
template <int SRC> __device__ __forceinline__ uint32_t mag_fold(uint32_t a, uint32_t b)
{
    return Src<SRC>::fold(a, b);
}

struct QuantArgs {
    const uint8_t *x;
    int64_t nbytes; // rows * cols * element size
    const float *fp8_scale;
    int rows, cols;
    const float *static_amax;
    uint8_t *codes, *sf_swz, *sf_lin;
    float *global_scale;
    const float *partials; // one max |x| per amax CTA (dynamic amax)
    float *slots;          // the fused kernels' grid exchange: one slot per CTA (same workspace)
    GridBarrier *barrier;  // ... and the launch's grid barrier (library-owned)
    int npartials;
    uint32_t nb_magic;     // ceil(2^32 / blocks per row): block / nb by multiply-high
    uint32_t runs_magic;   // ceil(2^32 / runs) for runs >= 2: item / runs by multiply-high
    int blocks_fit32;      // rows * blocks per row < 2^32 (the multiply-high path applies)
    int *status;
};

// K1: max |x| over a contiguous byte range per CTA, streamed through a shared-memory ring
// with 1-D bulk copies; one partial per CTA. `bid` / `nblk`: this CTA's index among the CTAs
// that share the tensor, and their number (the whole grid for one tensor, a slice of it in a
// batch).
template <int SRC>
__device__ __forceinline__ void amax_body(const uint8_t *__restrict__ x, int64_t nbytes,
                                          float *__restrict__ partials, int *status, int bid,
                                          int nblk, uint8_t *ring)
{
    __shared__ uint64_t bars[kRing];
    __shared__ float s_red[kAmaxThreads / 32];
    // whole 16-byte vectors only (bulk copies move multiples of 16 bytes); a tensor's last
    // nbytes % 16 bytes are folded by the kernel that reads the partials
    const int64_t nvec = nbytes >> 4;
    const int64_t nfull = nvec << 4;
    const int64_t per = ((nvec + nblk - 1) / nblk) << 4;
    const int64_t b0 = min(nfull, per * (int64_t)bid);
    const int64_t b1 = min(nfull, b0 + per);
    const int nchunks = (int)((b1 - b0 + kChunk - 1) / kChunk);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i)
            mbar_init(&bars[i], 1);
        fence_barrier_init();
    }
    __syncthreads();
    auto issue = [&](int c) {
        const int64_t off = b0 + (int64_t)c * kChunk;
        const uint32_t n = (uint32_t)min((int64_t)kChunk, b1 - off);
        mbar_arrive_expect_tx(&bars[c % kRing], n);
        bulk_load_1d(ring + (c % kRing) * kChunk, x + off, n, &bars[c % kRing]);
    };
    if (threadIdx.x == 0)
        for (int c = 0; c < min(nchunks, kRing); ++c)
            issue(c);
    pdl_launch_dependents(); // the encode kernel may start its own loads meanwhile
    uint32_t m = 0;
    for (int c = 0; c < nchunks; ++c) {
        const int slot = c % kRing;
        if (!mbar_wait(&bars[slot], (uint32_t)(c / kRing) & 1u, kSpinLimit))
            atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
        const int nv = (int)(min((int64_t)kChunk, b1 - (b0 + (int64_t)c * kChunk)) >> 4);
        const uint32_t base = smem_u32(ring + slot * kChunk);
        for (int i = threadIdx.x; i < nv; i += kAmaxThreads)
            m = mag_fold<SRC>(m, Src<SRC>::vec_magmax(lds128(base + 16 * i)));
        __syncthreads(); // every thread is done with this slot
        if (threadIdx.x == 0 && c + kRing < nchunks)
            issue(c + kRing);
    }
    float f = Src<SRC>::mag_to_f32(m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    if ((threadIdx.x & 31) == 0)
        s_red[threadIdx.x >> 5] = f;
    __syncthreads();
    if (threadIdx.x < 32) {
        f = threadIdx.x < kAmaxThreads / 32 ? s_red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
        if (threadIdx.x == 0)
            partials[bid] = f;
    }
}

template <int SRC>
__global__ void __launch_bounds__(kAmaxThreads, 1)
    amax_kernel(const uint8_t *__restrict__ x, int64_t nbytes, float *__restrict__ partials,
                int *status)
{
    extern __shared__ __align__(128) uint8_t ring[];
    amax_body<SRC>(x, nbytes, partials, status, blockIdx.x, gridDim.x, ring);
}

// Geometry of the fused kernel's warp items: a lane owns kBpl whole blocks (2 for bf16 / fp8,
// 1 for fp32) of a 32 * kBpl-block item.
template <int SRC> struct Enc {
    static constexpr int kEsz = Src<SRC>::kBytes;
    static constexpr int kBlk = 16 * kEsz;                    // bytes per block
    static constexpr int kVecs = kBlk / 16;                   // 16-byte vectors per block
    static constexpr int kBpl = SRC == kSrcF32 ? 1 : 2;       // blocks per lane
    static constexpr int kItemBlocks = 32 * kBpl;
    static constexpr int kItem = kItemBlocks * kBlk;          // bytes per warp item
};

// Maxima of one block from its raw vectors (fp8: of |e|, before the fp8 scale).
template <int SRC> __device__ __forceinline__ float block_maximum(const uint4 *r)
{
    if constexpr (SRC == kSrcBF16)
        return block_absmax_bf16(r[0], r[1]);
    else if constexpr (SRC == kSrcF32)
        return block_absmax_f32(r);
    else
        return block_absmax_e4m3(r[0]);
}

// The two code words of one block from its raw vectors, times rcp (fp8: times s8 first); zero
// when the block's scale is zero.
template <int SRC>
__device__ __forceinline__ uint2 block_codes(const uint4 *r, float s8, uint32_t sb, float rcp)
{
    uint2 c;
    if constexpr (SRC == kSrcBF16) {
        c = make_uint2(codes8_bf16(r[0], rcp), codes8_bf16(r[1], rcp));
    } else if constexpr (SRC == kSrcF32) {
        c = make_uint2(codes4_f32(r[0], rcp) | (codes4_f32(r[1], rcp) << 16),
                       codes4_f32(r[2], rcp) | (codes4_f32(r[3], rcp) << 16));
    } else {
        c = make_uint2(codes8_e4m3(r[0].x, r[0].y, s8, rcp), codes8_e4m3(r[0].z, r[0].w, s8, rcp));
    }
    return sb != 0u ? c : make_uint2(0u, 0u);
}

// Scale bytes of two blocks with maxima m0, m1 (fp8: of |e|; the fp8 scale applied here):
// sb0 | sb1 << 8; all zero when sg is zero.
template <int SRC>
__device__ __forceinline__ uint32_t scales_of_pair(float m0, float m1, float s8, float sg, float t,
                                                   float rt)
{
    if (!(sg > 0.0f))
        return 0u;
    if constexpr (SRC == kSrcE4M3) { // max |e| * s8 == max |e * s8| (rounding is monotone)
        m0 = __fmul_rn(m0, s8);
        m1 = __fmul_rn(m1, s8);
    }
    return scale_pair(m0, m1, t, rt);
}

// Shared-memory reads of a lane's blocks in rotated order: lane reads its vector v ^ k at step v
// (k = (lane / 2) % 4 for bf16 / fp32 with 4 vectors a lane, (lane / 4) % 2 for fp8 with 2),
// so the 8 lanes of a quarter-warp hit 8 different 16-byte bank groups. r[v] then holds the
// lane's natural vector v ^ k.
template <int SRC> __device__ __forceinline__ uint32_t lane_rotation(int lane)
{
    return SRC == kSrcE4M3 ? (uint32_t)(lane >> 2) & 1u : (uint32_t)(lane >> 1) & 3u;
}

// Natural-order maxima of a lane's blocks from rotated vectors (see lane_rotation).
template <int SRC>
__device__ __forceinline__ void lane_maxima_rot(const uint4 *r, uint32_t k, float &m0, float &m1)
{
    if constexpr (SRC == kSrcF32) {
        m0 = block_absmax_f32(r); // one block: the vector order does not matter
        m1 = 0.0f;
    } else {
        constexpr int V = Enc<SRC>::kVecs;
        // a block's vectors stay together; the rotation's top bit swaps the two blocks
        const float ma = block_maximum<SRC>(r), mb = block_maximum<SRC>(r + V);
        const bool sw = SRC == kSrcE4M3 ? (k & 1u) != 0 : (k & 2u) != 0;
        m0 = sw ? mb : ma;
        m1 = sw ? ma : mb;
    }
}

// Scales and natural-order code words of a lane's blocks from rotated vectors and natural
// maxima: the codes are computed in the rotated order and put back in place with selects.
template <int SRC>
__device__ __forceinline__ void lane_encode_rot(const uint4 *r, uint32_t k, float m0, float m1,
                                                float s8, float sg, float t, float rt,
                                                const float *rcp_tab,
                                                uint32_t (&cw)[2 * Enc<SRC>::kBpl],
                                                uint32_t &sb0, uint32_t &sb1)
{
    if constexpr (SRC == kSrcF32) {
        sb0 = sg > 0.0f ? e4m3_of_quotient(m0, t, rt) : 0u;
        sb1 = 0u;
        const float rcp = rcp_tab[sb0];
        uint32_t h[4]; // h[v]: codes of natural vector v ^ k
#pragma unroll
        for (int v = 0; v < 4; ++v)
            h[v] = codes4_f32(r[v], rcp);
        const bool b0 = (k & 1u) != 0, b1 = (k & 2u) != 0;
        const uint32_t d0 = b0 ? h[1] : h[0], d1 = b0 ? h[0] : h[1];
        const uint32_t d2 = b0 ? h[3] : h[2], d3 = b0 ? h[2] : h[3];
        const uint32_t o0 = b1 ? d2 : d0, o1 = b1 ? d3 : d1, o2 = b1 ? d0 : d2, o3 = b1 ? d1 : d3;
        cw[0] = sb0 ? (o0 | (o1 << 16)) : 0u;
        cw[1] = sb0 ? (o2 | (o3 << 16)) : 0u;
    } else {
        constexpr int V = Enc<SRC>::kVecs;
        const uint32_t s2 = scales_of_pair<SRC>(m0, m1, s8, sg, t, rt);
        sb0 = s2 & 0xFFu;
        sb1 = s2 >> 8;
        const bool sw = SRC == kSrcE4M3 ? (k & 1u) != 0 : (k & 2u) != 0;
        const uint32_t sa = sw ? sb1 : sb0, sbb = sw ? sb0 : sb1; // scales of r[0..V), r[V..2V)
        uint2 ca = block_codes<SRC>(r, s8, sa, rcp_tab[sa]);
        uint2 cb = block_codes<SRC>(r + V, s8, sbb, rcp_tab[sbb]);
        if constexpr (SRC == kSrcBF16) { // within a block, the rotation's low bit swaps halves
            if (k & 1u) {
                ca = make_uint2(ca.y, ca.x);
                cb = make_uint2(cb.y, cb.x);
            }
        }
        cw[0] = sw ? cb.x : ca.x;
        cw[1] = sw ? cb.y : ca.y;
        cw[2] = sw ? ca.x : cb.x;
        cw[3] = sw ? ca.y : cb.y;
    }
}

// Store a lane's codes (blocks f0 .. f0 + kBpl - 1) and scales in the linear and / or
// swizzled layout; the lane holding a row's last blocks also zeroes the atom's padding.
template <int SRC>
__device__ __forceinline__ void store_lane(const QuantArgs &a, int64_t f0, uint32_t nb, int apb,
                                           const uint32_t (&cw)[2 * Enc<SRC>::kBpl],
                                           uint32_t sb0, uint32_t sb1)
{
    uint8_t *cp = a.codes + f0 * 8;
    if constexpr (Enc<SRC>::kBpl == 2)
        *reinterpret_cast<uint4 *>(cp) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    else
        *reinterpret_cast<uint2 *>(cp) = make_uint2(cw[0], cw[1]);
    uint32_t row, b;
    if (a.blocks_fit32) {
        row = __umulhi((uint32_t)f0, a.nb_magic);
        if (row * nb > (uint32_t)f0)
            --row;
        b = (uint32_t)f0 - row * nb;
    } else {
        row = (uint32_t)(f0 / nb);
        b = (uint32_t)(f0 - (int64_t)row * nb);
    }
    const int64_t swz = ((int64_t)(row >> 7) * apb + (b >> 2)) * 512 + ((row & 31) << 4) +
                        (((row >> 5) & 3) << 2) + (b & 3);
    if constexpr (Enc<SRC>::kBpl == 2) {
        // b is even: both scale bytes are adjacent in either layout
        const uint16_t s2 = (uint16_t)(sb0 | (sb1 << 8));
        if (a.sf_lin)
            *reinterpret_cast<uint16_t *>(a.sf_lin + f0) = s2;
        if (a.sf_swz) {
            if (b + 2 == nb && (b & 3) == 0) // last pair of the row: zero the atom's pad
                *reinterpret_cast<uint32_t *>(a.sf_swz + swz) = s2;
            else
                *reinterpret_cast<uint16_t *>(a.sf_swz + swz) = s2;
        }
    } else {
        if (a.sf_lin)
            a.sf_lin[f0] = (uint8_t)sb0;
        if (a.sf_swz) {
            a.sf_swz[swz] = (uint8_t)sb0;
            if (b + 1 == nb && (b & 3) == 1) { // last block of the row: zero the pad
                a.sf_swz[swz + 1] = 0;
                a.sf_swz[swz + 2] = 0;
            }
        }
    }
}

// Zero the swizzled padding rows of the last 128-row band. In an atom, the 16-byte line
// i holds rows i, i + 32, i + 64, i + 96 of the band (4 bytes each), so one warp covers an
// atom with one store per lane: 16 bytes when all four rows are padding, else only the
// padding rows' words (the real rows' words belong to the encoding lanes). The pad blocks of
// real rows are written with their row's last scales.
__device__ __forceinline__ void zero_pad_rows(const QuantArgs &a, int apb, int bid, int nblk)
{
    if (!a.sf_swz || (a.rows & 127) == 0)
        return;
    const int band = a.rows >> 7;     // the partly filled band
    const int real = a.rows & 127;    // its real rows
    const int i = threadIdx.x & 31;   // line of the atom
    const int warps = blockDim.x >> 5;
    for (int atom = bid * warps + (threadIdx.x >> 5); atom < apb; atom += nblk * warps) {
        uint8_t *line = a.sf_swz + ((int64_t)band * apb + atom) * 512 + i * 16;
        if (i >= real) {
            *reinterpret_cast<uint4 *>(line) = make_uint4(0u, 0u, 0u, 0u);
        } else {
#pragma unroll
            for (int q = 1; q < 4; ++q)
                if (i + 32 * q >= real)
                    *reinterpret_cast<uint32_t *>(line + 4 * q) = 0u;
        }
    }
}

__device__ __forceinline__ uint4 ldg_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// K2: encode (tensors above the fused kernel's size). One CTA per SM owns a contiguous range
// of rows; each warp takes a 64-block run of one row and each lane two adjacent 16-value
// blocks, so address arithmetic and loop control are shared by two blocks, the codes leave as
// one 16-byte store and the two scale bytes as one 16-bit store. The first item is loaded
// before waiting on the amax kernel (programmatic dependent launch), so the loads overlap its
// tail; later items are double-buffered.
template <int SRC, int NT = kEncThreads>
__device__ __forceinline__ void encode_body(const QuantArgs &a, int bid, int nblk)
{
    __shared__ float s_sg;
    __shared__ float s_rcp[128];
    constexpr int kBlkBytes = 16 * Src<SRC>::kBytes;
    constexpr int V = Enc<SRC>::kVecs; // 16-byte vectors per block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = a.cols >> 4;       // blocks per row
    const int runs = (nb + 63) >> 6;  // 64-block runs per row (one per warp item)
    const int apb = (nb + 3) >> 2;    // scale atoms per 128-row band
    const int64_t row_bytes = (int64_t)a.cols * Src<SRC>::kBytes;
    const int r0 = (int)((int64_t)a.rows * bid / nblk);
    const int r1 = (int)((int64_t)a.rows * (bid + 1) / nblk);
    const int items = (r1 - r0) * runs;
    const uint8_t *xbase = a.x + (int64_t)r0 * row_bytes;

    // item -> (row offset, first block of this lane). Items are taken from the end of the
    // CTA's rows backwards: the amax pass read the tensor front to back, so the last part of
    // each CTA's range is the part still in L2 (for tensors too large for the fused kernel
    // most of the re-read then hits L2). The quotient by multiply-high is exact or one too
    // large (item < 2^31, runs < 2^26); one correction.
    auto item_rb = [&](int it_fwd, int &ro, int &b0) {
        if (it_fwd >= items) { // past this CTA's items: nothing to load or store
            ro = 0;
            b0 = nb;
            return;
        }
        const int it = items - 1 - it_fwd;
        if (runs == 1) {
            ro = it;
            b0 = 2 * lane;
            return;
        }
        ro = (int)__umulhi((uint32_t)it, a.runs_magic);
        if (ro * runs > it)
            --ro;
        b0 = (it - ro * runs) * 64 + 2 * lane;
    };
    // the lane's two blocks are contiguous in memory: 2 * V vectors
    auto load_item = [&](int it, uint4 (&r)[8], int &ro, int &b0) {
        item_rb(it, ro, b0);
        if (it < items && b0 < nb) {
            const uint4 *q =
                reinterpret_cast<const uint4 *>(xbase + (int64_t)ro * row_bytes + b0 * kBlkBytes);
            const int nv = b0 + 1 < nb ? 2 * V : V;
#pragma unroll
            for (int v = 0; v < 2 * V; ++v)
                if (v < nv)
                    r[v] = ldg_stream(q + v);
        }
    };

    int it = warp;
    uint4 ra[8], rb[8];
    int roa, b0a, rob, b0b;
    load_item(it, ra, roa, b0a);

    const float s8 = (SRC == kSrcE4M3 && a.fp8_scale) ? *a.fp8_scale : 1.0f;
    if (!a.static_amax)
        pdl_wait(); // the amax kernel's partial maxima are complete and visible
    if (threadIdx.x < 32) {
        float g = 0.0f;
        if (a.static_amax) {
            g = *a.static_amax;
        } else {
            // up to 8 loads in flight per lane: one L2 round trip per 256 partials
            for (int i0 = 0; i0 < a.npartials; i0 += 32 * 8) {
                float pv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + threadIdx.x + 32 * u;
                    pv[u] = i < a.npartials ? __ldcg(a.partials + i) : 0.0f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    g = fmaxf(g, pv[u]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
            if (SRC == kSrcE4M3)
                g = __fmul_rn(g, s8); // max |e| * s8 == max |e * s8| (rounding is monotone)
        }
        if (threadIdx.x == 0) {
            const float sg = __fdiv_rn(g, 2688.0f); // 6 * 448
            s_sg = sg;
            if (bid == 0)
                *a.global_scale = sg;
        }
    }
    __syncthreads();
    const float sg = s_sg;
    const float t = __fmul_rn(sg, 6.0f);
    const float rt = __frcp_rn(t);
    if (threadIdx.x < 128)
        s_rcp[threadIdx.x] = __frcp_rn(__fmul_rn(e4m3_to_f32(threadIdx.x), sg));
    __syncthreads();
    pdl_launch_dependents(); // a dependent GEMM may set up while this grid encodes

    // blocks b0, b0 + 1 of row r0 + ro: codes, scales; atom padding blocks get zero scales
    auto encode_store = [&](int ro, int b0, const uint4 (&r)[8]) {
        const int row = r0 + ro;
        uint32_t sb0 = 0, sb1 = 0;
        if (b0 < nb) {
            // b0 is even and nb is even (cols % 32 == 0): both blocks lie in the row
            const uint32_t s2 = scales_of_pair<SRC>(block_maximum<SRC>(r),
                                                    block_maximum<SRC>(r + V), s8, sg, t, rt);
            sb0 = s2 & 0xFFu;
            sb1 = s2 >> 8;
            const uint2 c0 = block_codes<SRC>(r, s8, sb0, s_rcp[sb0]);
            const uint2 c1 = block_codes<SRC>(r + V, s8, sb1, s_rcp[sb1]);
            uint8_t *c = a.codes + (int64_t)row * (a.cols >> 1) + b0 * 8;
            *reinterpret_cast<uint4 *>(c) = make_uint4(c0.x, c0.y, c1.x, c1.y);
            if (a.sf_lin) {
                uint8_t *l = a.sf_lin + (int64_t)row * nb + b0;
                if (b0 + 1 < nb)
                    *reinterpret_cast<uint16_t *>(l) = (uint16_t)(sb0 | (sb1 << 8));
                else
                    *l = (uint8_t)sb0;
            }
        }
        if (a.sf_swz && b0 < 4 * apb) // b0 even: both bytes in one atom, adjacent
            *reinterpret_cast<uint16_t *>(
                a.sf_swz + ((int64_t)(row >> 7) * apb + (b0 >> 2)) * 512 + ((row & 31) << 4) +
                (((row >> 5) & 3) << 2) + (b0 & 3)) = (uint16_t)(sb0 | (sb1 << 8));
    };
    if constexpr (SRC == kSrcF32) {
        // fp32 blocks are 64 bytes: one item in flight keeps the registers in budget
        while (it < items) {
            encode_store(roa, b0a, ra);
            it += NT / 32;
            load_item(it, ra, roa, b0a);
        }
    } else {
        while (it < items) {
            load_item(it + NT / 32, rb, rob, b0b);
            encode_store(roa, b0a, ra);
            it += NT / 32;
            if (it >= items)
                break;
            load_item(it + NT / 32, ra, roa, b0a);
            encode_store(rob, b0b, rb);
            it += NT / 32;
        }
    }
    zero_pad_rows(a, apb, bid, nblk);
}

template <int SRC>
__global__ void __launch_bounds__(kEncThreads, 1) encode_kernel(const QuantArgs a)
{
    encode_body<SRC>(a, blockIdx.x, gridDim.x);
}

// Fused single-pass quantizer for tensors that fit in the CTAs' shared memory (one CTA per
// SM, up to kFusedCap bytes each): each CTA bulk-loads its contiguous share of warp items in
// 32 KB copies. Dynamic amax: it folds max |x| over its share as the copies land, publishes
// one partial, meets the other CTAs at the library's bounded grid-wide barrier (cooperative
// launch: all CTAs are co-resident; grid_exchange.cuh), reduces the partials to the global
// scale and encodes from shared memory, so
// the tensor is read from HBM once and no second kernel is launched. Static amax: no
// barrier, each item is encoded as soon as its copy lands. Each lane reads its 64 (fp8: 32)
// contiguous bytes as 16-byte vectors in a rotated order (lane_rotation): conflict-free.
//
// With SS >= 0 the same launch also quantizes a second, smaller tensor b (source type SS)
// that is held in registers: each CTA takes a contiguous range of b's blocks, every thread
// loads whole blocks of it (kPairRegVecs 16-byte vectors: 4 blocks of fp8, 2 of bf16, 1 of
// fp32) with plain loads issued right after a's bulk copies, folds max |b| as they arrive,
// keeps them across the grid-wide barrier (b's partials meet a's there) and encodes them
// before a's shared-memory encode. Two tensors then cost one launch, one barrier and one HBM
// read each, with all of both in flight at once (nvfp4_quantize_batch of, e.g., a layer's FP8
// weight and its activations). Measured on W 3072x3072 FP8 + X 4096x3072 bf16 (globaltimer
// stamps in an instrumented copy, with the earlier cooperative-groups barrier): loads and
// maxima ~7-8 us, grid barrier ~2 us (the library's own one-atomic barrier takes ~1 us),
// partials + W's encode ~6 us, X's encode ~3.5 us; 1024 threads x 4 vectors beat 768 x 6 by
// ~0.5 us.
constexpr int kPairThreads = 1024; // 64 registers a thread: b's 16 plus the encode's
constexpr int kPairRegVecs = 4;

// b's part of the pair kernel after the grid-wide barrier and its global scale sg: each
// thread's register-held blocks encoded and stored (codes 8 bytes a block; scales in the linear
// and / or swizzled layout, a row's last atom padded with zeros; padding rows of the last band
// zeroed). rcp_tab: 1 / (E4M3(c) * sg) for the 128 non-negative codes.
template <int SS, int BPT>
__device__ __forceinline__ void pair_encode_regs(const QuantArgs &b, const uint4 *bv, int64_t bk0,
                                                 int64_t bk1, float s8, float sg,
                                                 const float *rcp_tab)
{
    constexpr int BV = Enc<SS>::kVecs;
    const float t = __fmul_rn(sg, 6.0f);
    const float rt = __frcp_rn(t);
    const uint32_t nb = (uint32_t)(b.cols >> 4);
    const int apb = (int)((nb + 3) >> 2);
    // two blocks at a time: their scales with one pair conversion (blocks past the range were
    // loaded as zeros)
    constexpr int STEP = BPT >= 2 ? 2 : 1;
#pragma unroll
    for (int j0 = 0; j0 < BPT; j0 += STEP) {
        uint32_t sbs[STEP];
        if constexpr (STEP == 2) {
            const uint32_t s2 = scales_of_pair<SS>(block_maximum<SS>(bv + j0 * BV),
                                                   block_maximum<SS>(bv + (j0 + 1) * BV), s8, sg,
                                                   t, rt);
            sbs[0] = s2 & 0xFFu;
            sbs[1] = s2 >> 8;
        } else {
            sbs[0] = sg > 0.0f ? e4m3_of_quotient(block_maximum<SS>(bv + j0 * BV), t, rt) : 0u;
        }
#pragma unroll
        for (int jj = 0; jj < STEP; ++jj) {
            const int j = j0 + jj;
            const int64_t blk = bk0 + (int64_t)j * blockDim.x + threadIdx.x;
            if (blk >= bk1)
                continue;
            const uint32_t sb = sbs[jj];
            const uint2 codes = block_codes<SS>(bv + j * BV, s8, sb, rcp_tab[sb]);
            *reinterpret_cast<uint2 *>(b.codes + blk * 8) = codes;
            if (b.sf_lin)
                b.sf_lin[blk] = (uint8_t)sb;
            if (b.sf_swz) {
                uint32_t row, c; // blk / nb by multiply-high (exact or one too large)
                if (b.blocks_fit32) {
                    row = __umulhi((uint32_t)blk, b.nb_magic);
                    if (row * nb > (uint32_t)blk)
                        --row;
                    c = (uint32_t)blk - row * nb;
                } else {
                    row = (uint32_t)(blk / nb);
                    c = (uint32_t)(blk - (int64_t)row * nb);
                }
                uint8_t *q = b.sf_swz + swz_offset(row, c, apb);
                q[0] = (uint8_t)sb;
                if (c + 1 == nb) // the row's last block: the rest of its atom row is padding
                    for (uint32_t e = (c & 3u) + 1u; e < 4u; ++e)
                        q[e - (c & 3u)] = 0u;
            }
        }
    }
    zero_pad_rows(b, apb, blockIdx.x, gridDim.x);
}

template <int SRC, int NT, int SS>
__device__ __forceinline__ void fused_body(const QuantArgs &a, const QuantArgs &b, uint8_t *buf)
{
    using E = Enc<SRC>;
    constexpr bool kPair = SS >= 0;
    // launched with programmatic dependent launch: set-up may overlap the previous kernel's
    // tail; nothing it writes is touched before this wait
    pdl_wait();
    __shared__ uint64_t bars[kFusedMaxChunks];
    __shared__ float s_red[NT / 32];
    __shared__ float s_red_b[NT / 32];
    __shared__ float s_sg, s_sgb;
    __shared__ float s_rcp[128];
    __shared__ float s_rcpb[kPair ? 128 : 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nblocks = (int64_t)a.rows * (a.cols >> 4);
    const int64_t nitems = (nblocks + E::kItemBlocks - 1) / E::kItemBlocks;
    const int64_t c0 = nitems * blockIdx.x / gridDim.x;
    const int64_t c1 = nitems * (blockIdx.x + 1) / gridDim.x;
    const int64_t byte0 = c0 * E::kItem;
    const int64_t nbytes = max((int64_t)0, min(a.nbytes, c1 * E::kItem) - byte0);
    const int nch = (int)((nbytes + kFusedChunk - 1) / kFusedChunk);
    // b's blocks: a contiguous range per CTA, block j * NT + tid of it per thread
    using EB = Enc<kPair ? SS : SRC>;
    constexpr int BV = EB::kVecs;                 // 16-byte vectors per block of b
    constexpr int BPT = kPairRegVecs / BV;        // b's blocks per thread
    const int64_t b_nblk = kPair ? (int64_t)b.rows * (b.cols >> 4) : 0;
    const int64_t b_per = (b_nblk + gridDim.x - 1) / gridDim.x;
    const int64_t bk0 = min(b_nblk, b_per * (int64_t)blockIdx.x);
    const int64_t bk1 = min(b_nblk, bk0 + b_per);
    const bool b_dyn = kPair && !b.static_amax;
    uint4 bv[kPair ? kPairRegVecs : 1];
    __shared__ float s_scalars[4];
    if (threadIdx.x == 0) {
        // the scalar inputs go out ahead of the bulk copies, not behind them in the queue
        s_scalars[0] = (SRC == kSrcE4M3 && a.fp8_scale) ? *a.fp8_scale : 1.0f;
        s_scalars[1] = a.static_amax ? *a.static_amax : 0.0f;
        if constexpr (kPair) {
            s_scalars[2] = (SS == kSrcE4M3 && b.fp8_scale) ? *b.fp8_scale : 1.0f;
            s_scalars[3] = b.static_amax ? *b.static_amax : 0.0f;
        }
        for (int i = 0; i < nch; ++i)
            mbar_init(&bars[i], 1);
        fence_barrier_init();
        for (int i = 0; i < nch; ++i) {
            const int64_t off = (int64_t)i * kFusedChunk;
            const uint32_t n = (uint32_t)min((int64_t)kFusedChunk, nbytes - off);
            mbar_arrive_expect_tx(&bars[i], n);
            bulk_load_1d(buf + off, a.x + byte0 + off, n, &bars[i]);
        }
    }
    if constexpr (kPair) {
        // all of this thread's blocks of b in flight at once
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
            const int64_t blk = bk0 + (int64_t)j * NT + threadIdx.x;
            const uint4 *q = reinterpret_cast<const uint4 *>(b.x + blk * EB::kBlk);
#pragma unroll
            for (int v = 0; v < BV; ++v)
                bv[j * BV + v] = blk < bk1 ? ldg_stream(q + v) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();
    const float s8 = s_scalars[0];
    const uint32_t k = lane_rotation<SRC>(lane);
    constexpr int NVL = E::kBpl * E::kVecs;
    constexpr int kWarps = NT / 32;
    constexpr int MIW = kFusedCap / E::kItem / kWarps; // items per warp at most
    const int items = (int)(c1 - c0);
    auto load_lane = [&](int j, uint4 (&r)[NVL]) -> bool {
        const int64_t f0 = (c0 + j) * E::kItemBlocks + lane * E::kBpl;
        const bool valid = f0 < nblocks;
        const uint32_t src = smem_u32(buf + j * E::kItem) + lane * (E::kBpl * E::kBlk);
#pragma unroll
        for (int v = 0; v < NVL; ++v)
            r[v] = valid ? lds128(src + 16 * (v ^ k)) : make_uint4(0u, 0u, 0u, 0u);
        return valid;
    };
    auto wait_item = [&](int j) {
        if (!mbar_wait(&bars[(j * E::kItem) / kFusedChunk], 0, kSpinLimit) && lane == 0)
            atomicExch(a.status, (int)NVFP4_ERR_TIMEOUT);
    };
    if constexpr (kPair) {
        // b's maxima first: its loads were issued right behind a's copies
        if (b_dyn) {
            uint32_t m = 0; // blocks past the range were loaded as zeros
#pragma unroll
            for (int i = 0; i < BPT * BV; ++i)
                m = mag_fold<SS>(m, Src<SS>::vec_magmax(bv[i]));
            float f = Src<SS>::mag_to_f32(m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
            if (lane == 0)
                s_red_b[warp] = f;
        }
    }
    const bool need_barrier = !a.static_amax || b_dyn;
    float bm0[MIW], bm1[MIW]; // block maxima of this lane's blocks, item by item
    if (!a.static_amax) {
        // block maxima as the copies land; the CTA maximum is their maximum
        float lm = 0.0f;
#pragma unroll
        for (int jj = 0; jj < MIW; ++jj) {
            const int j = warp + kWarps * jj;
            bm0[jj] = bm1[jj] = 0.0f;
            if (j < items) {
                wait_item(j);
                uint4 r[NVL];
                load_lane(j, r);
                lane_maxima_rot<SRC>(r, k, bm0[jj], bm1[jj]);
                lm = fmaxf(lm, fmaxf(bm0[jj], bm1[jj]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            lm = fmaxf(lm, __shfl_xor_sync(0xFFFFFFFFu, lm, o));
        if (lane == 0)
            s_red[warp] = lm;
    }
    // the global scales: every CTA's maxima of both tensors exchanged through the workspace
    // in one bounded grid-wide exchange (a single CTA already holds the maxima)
    if (need_barrier)
        __syncthreads();
    if (threadIdx.x < 32) {
        float g = 0.0f, gb = 0.0f;
        if (!a.static_amax) {
            g = threadIdx.x < kWarps ? s_red[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
        }
        if (b_dyn) {
            gb = threadIdx.x < kWarps ? s_red_b[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                gb = fmaxf(gb, __shfl_xor_sync(0xFFFFFFFFu, gb, o));
        }
        if (need_barrier && gridDim.x > 1) {
            float ga_all, gb_all;
            if (!grid_exchange_max(a.slots, a.barrier, (int)gridDim.x, (int)blockIdx.x, g, gb,
                                   kExchangeLimit, ga_all, gb_all) &&
                threadIdx.x == 0)
                atomicExch(a.status, (int)NVFP4_ERR_TIMEOUT);
            g = ga_all;
            gb = gb_all;
        }
        if (b_dyn && SS == kSrcE4M3)
            gb = __fmul_rn(gb, s_scalars[2]); // max |e| * s8 == max |e * s8|
        if (!a.static_amax && SRC == kSrcE4M3)
            g = __fmul_rn(g, s8); // max |e| * s8 == max |e * s8| (rounding is monotone)
        if (threadIdx.x == 0) {
            const float sg = __fdiv_rn(a.static_amax ? s_scalars[1] : g, 2688.0f); // 6 * 448
            s_sg = sg;
            if (blockIdx.x == 0)
                *a.global_scale = sg;
            if constexpr (kPair) {
                const float sgb = __fdiv_rn(b.static_amax ? s_scalars[3] : gb, 2688.0f);
                s_sgb = sgb;
                if (blockIdx.x == 0)
                    *b.global_scale = sgb;
            }
        }
    }
    __syncthreads();
    const float sg = s_sg;
    const float t = __fmul_rn(sg, 6.0f);
    const float rt = __frcp_rn(t);
    if (threadIdx.x < 128)
        s_rcp[threadIdx.x] = __frcp_rn(__fmul_rn(e4m3_to_f32(threadIdx.x), sg));
    if (kPair && threadIdx.x >= 128 && threadIdx.x < 256)
        s_rcpb[threadIdx.x - 128] = __frcp_rn(__fmul_rn(e4m3_to_f32(threadIdx.x - 128), s_sgb));
    __syncthreads();
    pdl_launch_dependents(); // a dependent GEMM may set up while this grid encodes
    if constexpr (kPair)
        pair_encode_regs<SS, BPT>(b, bv, bk0, bk1, s_scalars[2], s_sgb, s_rcpb);

    const uint32_t nb = (uint32_t)(a.cols >> 4);
    const int apb = (int)((nb + 3) >> 2);
#pragma unroll
    for (int jj = 0; jj < MIW; ++jj) {
        const int j = warp + kWarps * jj;
        if (j >= items)
            break;
        uint4 r[NVL];
        if (a.static_amax) { // the copy may still be in flight; maxima not taken yet
            wait_item(j);
            load_lane(j, r);
            lane_maxima_rot<SRC>(r, k, bm0[jj], bm1[jj]);
        } else {
            load_lane(j, r);
        }
        const int64_t f0 = (c0 + j) * E::kItemBlocks + lane * E::kBpl;
        uint32_t cw[2 * E::kBpl], sb0, sb1;
        lane_encode_rot<SRC>(r, k, bm0[jj], bm1[jj], s8, sg, t, rt, s_rcp, cw, sb0, sb1);
        if (f0 < nblocks)
            store_lane<SRC>(a, f0, nb, apb, cw, sb0, sb1);
    }
    zero_pad_rows(a, apb, blockIdx.x, gridDim.x);
}

template <int SRC>
__global__ void __launch_bounds__(kFusedThreads, 1) fused_quantize_kernel(const QuantArgs a)
{
    extern __shared__ __align__(128) uint8_t buf[];
    fused_body<SRC, kFusedThreads, -1>(a, a, buf);
}

// a held in shared memory, b streamed (see fused_body).
template <int SA, int SB>
__global__ void __launch_bounds__(kPairThreads, 1)
    fused_pair_quantize_kernel(const QuantArgs a, const QuantArgs b)
{
    extern __shared__ __align__(128) uint8_t buf[];
    fused_body<SA, kPairThreads, SB>(a, b, buf);
}

// Single-launch quantizer for tensors larger than the CTAs' shared memory. One CTA per SM owns
// a contiguous range of warp items and streams it through a ring of kStreamSlots chunks with
// 1-D bulk copies; a chunk holds kStreamIpw items per warp. Dynamic amax: pass 1 folds max |x|
// over the range front to back; the grid-wide exchange gives sg; pass 2 walks the range back
// to front, so it starts on the chunks pass 1 left in the ring (no second read) and continues
// on the ones read last, which L2 still holds; each warp encodes its items of the chunk (block
// maxima, E4M3 scales, E2M1 codes; the two items are independent, so their instructions
// interleave) and the chunk's slot is refilled with the chunk kStreamSlots further down. Static
// amax: pass 2 alone. The tensor leaves HBM once and one kernel runs. The encode is bound by
// the integer pipe, so the per-chunk bookkeeping is kept small: every wait's mbarrier parity
// is a closed form of the chunk index.
constexpr int kStreamThreads = 512;
constexpr int kStreamSlots = 3;
constexpr int kStreamIpw = 2; // warp items per warp per chunk

template <int SRC> struct StreamCfg {
    static constexpr int kWarps = kStreamThreads / 32;
    static constexpr int kChunkItems = kWarps * kStreamIpw;
    static constexpr int kChunkBytes = kChunkItems * Enc<SRC>::kItem; // 64 KB (fp8: 32 KB)
    static constexpr int kSmem = kStreamSlots * kChunkBytes;
};

// max |x| of one 16-byte vector folded into acc (bf16: packed magnitudes, sign bits not
// meaningful; fp32: the float; fp8: packed f16 magnitudes of |e|)
template <int SRC> __device__ __forceinline__ uint32_t fold_vec(uint32_t acc, const uint4 &v)
{
    if constexpr (SRC == kSrcBF16) {
        return absmax_bf16x2(acc, absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)));
    } else if constexpr (SRC == kSrcF32) {
        return __float_as_uint(fmaxf(__uint_as_float(acc),
                                     fmaxf(fmaxf(fabsf(__uint_as_float(v.x)),
                                                 fabsf(__uint_as_float(v.y))),
                                           fmaxf(fabsf(__uint_as_float(v.z)),
                                                 fabsf(__uint_as_float(v.w))))));
    } else {
        const uint32_t a0 = absmax_f16x2(e4m3x2_to_f16x2(v.x), e4m3x2_to_f16x2(v.x >> 16));
        const uint32_t a1 = absmax_f16x2(e4m3x2_to_f16x2(v.y), e4m3x2_to_f16x2(v.y >> 16));
        const uint32_t a2 = absmax_f16x2(e4m3x2_to_f16x2(v.z), e4m3x2_to_f16x2(v.z >> 16));
        const uint32_t a3 = absmax_f16x2(e4m3x2_to_f16x2(v.w), e4m3x2_to_f16x2(v.w >> 16));
        return absmax_f16x2(acc, absmax_f16x2(absmax_f16x2(a0, a1), absmax_f16x2(a2, a3)));
    }
}

// the folded value as an fp32 maximum (fp8: of |e|)
template <int SRC> __device__ __forceinline__ float fold_to_f32(uint32_t acc)
{
    if constexpr (SRC == kSrcBF16) {
        return fmaxf(__uint_as_float((acc << 16) & 0x7FFFFFFFu),
                     __uint_as_float(acc & 0x7FFF0000u));
    } else if constexpr (SRC == kSrcF32) {
        return __uint_as_float(acc);
    } else {
        __half_raw lo, hi;
        lo.x = (unsigned short)(acc & 0x7FFFu);
        hi.x = (unsigned short)((acc >> 16) & 0x7FFFu);
        return fmaxf(__half2float(__half(lo)), __half2float(__half(hi)));
    }
}

template <int SRC>
__global__ void __launch_bounds__(kStreamThreads, 1) stream_quantize_kernel(const QuantArgs a)
{
    using E = Enc<SRC>;
    using C = StreamCfg<SRC>;
    constexpr int S = kStreamSlots;
    constexpr int NVL = E::kBpl * E::kVecs; // 16-byte vectors of a lane's blocks
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t full[S];
    __shared__ float s_red[C::kWarps];
    __shared__ float s_sg;
    __shared__ float s_rcp[128];
    pdl_wait(); // the tensor and the outputs belong to the stream's earlier work
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t k = lane_rotation<SRC>(lane);
    const bool dyn = a.static_amax == nullptr;
    const int64_t nblocks = (int64_t)a.rows * (a.cols >> 4);
    const int64_t nitems = (nblocks + E::kItemBlocks - 1) / E::kItemBlocks;
    const int64_t c0 = nitems * blockIdx.x / gridDim.x;
    const int64_t c1 = nitems * (blockIdx.x + 1) / gridDim.x;
    const int64_t byte0 = c0 * E::kItem;
    const int64_t nbytes = max((int64_t)0, min(a.nbytes, c1 * E::kItem) - byte0);
    const int nch = (int)((nbytes + C::kChunkBytes - 1) / C::kChunkBytes);
    const float s8 = (SRC == kSrcE4M3 && a.fp8_scale) ? *a.fp8_scale : 1.0f;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s)
            mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    auto issue = [&](int c) { // thread 0 only
        const int64_t off = (int64_t)c * C::kChunkBytes;
        const uint32_t n = (uint32_t)min((int64_t)C::kChunkBytes, nbytes - off);
        mbar_arrive_expect_tx(&full[c % S], n);
        bulk_load_1d(ring + (c % S) * C::kChunkBytes, a.x + byte0 + off, n, &full[c % S]);
    };
    auto wait_chunk = [&](int c, uint32_t parity) {
        if (!mbar_wait(&full[c % S], parity, kSpinLimit) && lane == 0)
            atomicExch(a.status, (int)NVFP4_ERR_TIMEOUT);
    };

    float g = 0.0f;
    if (dyn) {
        // pass 1: max |x| over the range, front to back; chunk c is fill c / S of its slot
        if (threadIdx.x == 0)
            for (int c = 0; c < min(nch, S); ++c)
                issue(c);
        uint32_t m = 0;
        for (int c = 0; c < nch; ++c) {
            wait_chunk(c, (uint32_t)(c / S) & 1u);
            const int nv = (int)(min((int64_t)C::kChunkBytes, nbytes - (int64_t)c * C::kChunkBytes) >> 4);
            const uint32_t base = smem_u32(ring + (c % S) * C::kChunkBytes);
            for (int i = threadIdx.x; i < nv; i += kStreamThreads)
                m = fold_vec<SRC>(m, lds128(base + 16 * i));
            if (c + S < nch) {
                __syncthreads(); // every thread is done with the slot
                if (threadIdx.x == 0)
                    issue(c + S);
            }
        }
        float f = fold_to_f32<SRC>(m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
        if (lane == 0)
            s_red[warp] = f;
        __syncthreads();
        if (warp == 0) {
            g = lane < C::kWarps ? s_red[lane] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
            if (gridDim.x > 1) {
                float unused;
                if (!grid_exchange_max(a.slots, a.barrier, (int)gridDim.x, (int)blockIdx.x, g,
                                       0.0f, kExchangeLimit, g, unused) &&
                    lane == 0)
                    atomicExch(a.status, (int)NVFP4_ERR_TIMEOUT);
            }
            if (SRC == kSrcE4M3)
                g = __fmul_rn(g, s8); // max |e| * s8 == max |e * s8| (rounding is monotone)
        }
    } else {
        // static amax: the last chunks first (pass 2's order)
        if (threadIdx.x == 0)
            for (int c = nch - 1; c >= max(0, nch - S); --c)
                issue(c);
        if (warp == 0)
            g = *a.static_amax;
    }
    if (threadIdx.x == 0) {
        const float sg = __fdiv_rn(g, 2688.0f); // 6 * 448
        s_sg = sg;
        if (blockIdx.x == 0)
            *a.global_scale = sg;
    }
    __syncthreads();
    const float sg = s_sg;
    const float t = __fmul_rn(sg, 6.0f);
    const float rt = __frcp_rn(t);
    if (threadIdx.x < 128)
        s_rcp[threadIdx.x] = __frcp_rn(__fmul_rn(e4m3_to_f32(threadIdx.x), sg));
    __syncthreads();
    pdl_launch_dependents(); // a dependent GEMM may set up while this grid encodes

    // pass 2: encode, back to front. A chunk below nch - S is a refill: with dynamic amax its
    // fill number is n1(s) + (nch - S - 1 - c) / S, n1(s) = (nch - 1 - s) / S + 1 fills of
    // slot s = c % S in pass 1; with a static amax it is 1 + (nch - S - 1 - c) / S (each slot's
    // first fill holds one of the last S chunks, waited with parity 0).
    const uint32_t nb = (uint32_t)(a.cols >> 4);
    const int apb = (int)((nb + 3) >> 2);
    for (int c = nch - 1; c >= 0; --c) {
        if (c < nch - S) {
            const int fill = dyn ? (nch - 1 - c % S) / S + 1 + (nch - S - 1 - c) / S
                                 : 1 + (nch - S - 1 - c) / S;
            wait_chunk(c, (uint32_t)fill & 1u);
        } else if (!dyn) {
            wait_chunk(c, 0u);
        }
        const uint32_t slot = smem_u32(ring + (c % S) * C::kChunkBytes);
#pragma unroll
        for (int h = 0; h < kStreamIpw; ++h) {
            const int w = warp + C::kWarps * h; // item of the chunk
            const int64_t item = c0 + (int64_t)c * C::kChunkItems + w;
            const int64_t f0 = item * E::kItemBlocks + lane * E::kBpl;
            if (item < c1 && f0 < nblocks) {
                const uint32_t src = slot + w * E::kItem + lane * (E::kBpl * E::kBlk);
                uint4 r[NVL];
#pragma unroll
                for (int v = 0; v < NVL; ++v)
                    r[v] = lds128(src + 16 * (v ^ k));
                float m0, m1;
                lane_maxima_rot<SRC>(r, k, m0, m1);
                uint32_t cw[2 * E::kBpl], sb0, sb1;
                lane_encode_rot<SRC>(r, k, m0, m1, s8, sg, t, rt, s_rcp, cw, sb0, sb1);
                store_lane<SRC>(a, f0, nb, apb, cw, sb0, sb1);
            }
        }
        if (c - S >= 0) {
            __syncthreads(); // every warp is done with the slot
            if (threadIdx.x == 0)
                issue(c - S);
        }
    }
    zero_pad_rows(a, apb, blockIdx.x, gridDim.x);
}

template <int SRC>
cudaError_t launch_typed(const void *x, const float *fp8_scale, int64_t rows, int64_t cols,
                         const float *static_amax, uint8_t *codes, uint8_t *sf_swz,
                         uint8_t *sf_lin, float *global_scale, void *ws, cudaStream_t s)
{
    const int sms = num_sms();
    QuantArgs qa{};
    qa.x = reinterpret_cast<const uint8_t *>(x);
    qa.fp8_scale = fp8_scale;
    qa.rows = (int)rows;
    qa.cols = (int)cols;
    qa.static_amax = static_amax;
    qa.codes = codes;
    qa.sf_swz = sf_swz;
    qa.sf_lin = sf_lin;
    qa.global_scale = global_scale;
    qa.partials = reinterpret_cast<const float *>(ws);
    qa.nbytes = rows * cols * Src<SRC>::kBytes;
    const uint64_t nb = (uint64_t)(cols / 16);
    qa.nb_magic = nb > 1 ? (uint32_t)((((uint64_t)1 << 32) + nb - 1) / nb) : 0u;
    qa.blocks_fit32 = (uint64_t)rows * nb < ((uint64_t)1 << 32) ? 1 : 0;
    const uint64_t runs = (nb + 63) / 64;
    qa.runs_magic = runs > 1 ? (uint32_t)((((uint64_t)1 << 32) + runs - 1) / runs) : 0u;
    qa.status = device_status_ptr();
    qa.slots = reinterpret_cast<float *>(ws);
    // fused single pass when every CTA's share fits in its shared memory
    {
        using E = Enc<SRC>;
        const int64_t nitems = (rows * (cols / 16) + E::kItemBlocks - 1) / E::kItemBlocks;
        int64_t g = (nitems + kFusedThreads / 32 - 1) / (kFusedThreads / 32);
        if (g > sms)
            g = sms;
        if (g < 1)
            g = 1;
        if ((nitems + g - 1) / g * E::kItem <= kFusedCap && g <= kExchangeMaxCtas &&
            qa.nbytes >= kFusedMinBytes) {
            if (!static_amax && !(qa.barrier = grid_barrier_for(s)))
                return cudaErrorInvalidValue;
            static std::once_flag fattr[64];
            int dev = 0;
            cudaGetDevice(&dev);
            cudaError_t fe = cudaSuccess;
            std::call_once(fattr[dev & 63], [&]() {
                fe = cudaFuncSetAttribute(fused_quantize_kernel<SRC>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedCap);
            });
            if (fe != cudaSuccess)
                return fe;
            cudaLaunchConfig_t fc{};
            fc.gridDim = dim3((unsigned)g);
            fc.blockDim = dim3(kFusedThreads);
            fc.dynamicSmemBytes = kFusedCap;
            fc.stream = s;
            cudaLaunchAttribute fa[2];
            fa[0].id = cudaLaunchAttributeCooperative;
            fa[0].val.cooperative = static_amax ? 0 : 1;
            fa[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            fa[1].val.programmaticStreamSerializationAllowed = 1;
            fc.attrs = fa;
            fc.numAttrs = 2;
            return cudaLaunchKernelEx(&fc, fused_quantize_kernel<SRC>, qa);
        }
        // larger tensors: one streamed launch (two passes through a shared-memory ring)
        if (qa.nbytes >= kFusedMinBytes && sms <= kExchangeMaxCtas) {
            if (!static_amax && !(qa.barrier = grid_barrier_for(s)))
                return cudaErrorInvalidValue;
            static std::once_flag sattr[64];
            int dev = 0;
            cudaGetDevice(&dev);
            cudaError_t se = cudaSuccess;
            std::call_once(sattr[dev & 63], [&]() {
                se = cudaFuncSetAttribute(stream_quantize_kernel<SRC>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          StreamCfg<SRC>::kSmem);
            });
            if (se != cudaSuccess)
                return se;
            cudaLaunchConfig_t sc{};
            sc.gridDim = dim3((unsigned)sms);
            sc.blockDim = dim3(kStreamThreads);
            sc.dynamicSmemBytes = StreamCfg<SRC>::kSmem;
            sc.stream = s;
            cudaLaunchAttribute sa[2];
            sa[0].id = cudaLaunchAttributeCooperative;
            sa[0].val.cooperative = static_amax ? 0 : 1;
            sa[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            sa[1].val.programmaticStreamSerializationAllowed = 1;
            sc.attrs = sa;
            sc.numAttrs = 2;
            return cudaLaunchKernelEx(&sc, stream_quantize_kernel<SRC>, qa);
        }
    }
    cudaError_t e;
    if (!static_amax) {
        const int64_t nbytes = rows * cols * Src<SRC>::kBytes;
        int g = sms < kAmaxPartials ? sms : kAmaxPartials;
        const int64_t need = (nbytes + kChunk - 1) / kChunk;
        if (need < g)
            g = need < 1 ? 1 : (int)need;
        qa.npartials = g;
        const size_t smem = (size_t)kRing * kChunk;
        e = cudaFuncSetAttribute(amax_kernel<SRC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess)
            return e;
        amax_kernel<SRC><<<g, kAmaxThreads, smem, s>>>(reinterpret_cast<const uint8_t *>(x),
                                                       nbytes, reinterpret_cast<float *>(ws),
                                                       device_status_ptr());
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    int grid = sms;
    if (rows < grid)
        grid = rows < 1 ? 1 : (int)rows;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kEncThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = static_amax ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_kernel<SRC>, qa);
}


// ---------------------------------------------------------------------------------------
// Batched quantize: several tensors in one amax launch and one encode launch. The grid's
// CTAs are split over the tensors in proportion to their bytes; a CTA finds its tensor by
// its index and runs the single-tensor body on its share (its own partial maxima, its own
// global scale), so the tensors' memory traffic overlaps instead of running back to back.
// ---------------------------------------------------------------------------------------

struct QuantGroup {
    int njobs;
    int src[kMaxQuantJobs];
    int amax_cta0[kMaxQuantJobs + 1]; // amax CTAs of job j: [amax_cta0[j], amax_cta0[j + 1])
    int enc_cta0[kMaxQuantJobs + 1];  // encode CTAs of job j
    QuantArgs job[kMaxQuantJobs];
};

__device__ __forceinline__ int job_of(const int *cta0, int njobs)
{
    int j = 0;
    while (j + 1 < njobs && (int)blockIdx.x >= cta0[j + 1])
        ++j;
    return j;
}

__global__ void __launch_bounds__(kAmaxThreads, 1) amax_group_kernel(const __grid_constant__ QuantGroup g)
{
    extern __shared__ __align__(128) uint8_t ring[];
    const int j = job_of(g.amax_cta0, g.njobs);
    const QuantArgs &a = g.job[j];
    const int bid = blockIdx.x - g.amax_cta0[j], nblk = g.amax_cta0[j + 1] - g.amax_cta0[j];
    float *part = const_cast<float *>(a.partials);
    switch (g.src[j]) {
    case kSrcF32: amax_body<kSrcF32>(a.x, a.nbytes, part, a.status, bid, nblk, ring); break;
    case kSrcBF16: amax_body<kSrcBF16>(a.x, a.nbytes, part, a.status, bid, nblk, ring); break;
    default: amax_body<kSrcE4M3>(a.x, a.nbytes, part, a.status, bid, nblk, ring); break;
    }
}

__global__ void __launch_bounds__(kEncThreads, 1) encode_group_kernel(const __grid_constant__ QuantGroup g)
{
    const int j = job_of(g.enc_cta0, g.njobs);
    const QuantArgs &a = g.job[j];
    const int bid = blockIdx.x - g.enc_cta0[j], nblk = g.enc_cta0[j + 1] - g.enc_cta0[j];
    switch (g.src[j]) {
    case kSrcF32: encode_body<kSrcF32>(a, bid, nblk); break;
    case kSrcBF16: encode_body<kSrcBF16>(a, bid, nblk); break;
    default: encode_body<kSrcE4M3>(a, bid, nblk); break;
    }
}

template <int SRC> void fill_args(QuantArgs &qa, const QuantJob &jb)
{
    qa.x = reinterpret_cast<const uint8_t *>(jb.x);
    qa.fp8_scale = jb.fp8_scale;
    qa.rows = (int)jb.rows;
    qa.cols = (int)jb.cols;
    qa.static_amax = jb.static_amax;
    qa.codes = jb.codes;
    qa.sf_swz = jb.scales_swz;
    qa.sf_lin = jb.scales_lin;
    qa.global_scale = jb.global_scale;
    qa.nbytes = jb.rows * jb.cols * Src<SRC>::kBytes;
    const uint64_t nb = (uint64_t)(jb.cols / 16);
    qa.nb_magic = nb > 1 ? (uint32_t)((((uint64_t)1 << 32) + nb - 1) / nb) : 0u;
    qa.blocks_fit32 = (uint64_t)jb.rows * nb < ((uint64_t)1 << 32) ? 1 : 0;
    const uint64_t runs = (nb + 63) / 64;
    qa.runs_magic = runs > 1 ? (uint32_t)((((uint64_t)1 << 32) + runs - 1) / runs) : 0u;
    qa.status = device_status_ptr();
}

// Split `total` CTAs over jobs in proportion to weight[j] (0 = no CTA), at least one each,
// at most cap[j]; writes the prefix sums to cta0 and returns the CTA count.
int split_ctas(int n, const int64_t *weight, const int64_t *cap, int total, int *cta0)
{
    int64_t wsum = 0;
    for (int j = 0; j < n; ++j)
        wsum += weight[j];
    cta0[0] = 0;
    for (int j = 0; j < n; ++j) {
        int64_t c = 0;
        if (weight[j] > 0) {
            c = wsum > 0 ? (int64_t)total * weight[j] / wsum : 1;
            if (c < 1)
                c = 1;
            if (c > cap[j])
                c = cap[j];
        }
        cta0[j + 1] = cta0[j] + (int)c;
    }
    return cta0[n];
}
// ---------------------------------------------------------------------------------------
// FP8 E4M3 tensorwise quantization ("Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization
// Details": embed_tokens / lm_head in float8_e4m3fn, tensorwise, round-to-nearest): one fp32
// scale s = amax / 448 per tensor, code = sign(x) | E4M3(|x| / s) (RN of the IEEE quotient,
// ties to even, saturating; s == 0 gives sign-only codes). HBM-bound elementwise pass after
// the amax kernel (programmatic dependent launch): 8 values per thread-step, 16 or 32 bytes
// in, 8 bytes out, grid-stride over the flat tensor.
// ---------------------------------------------------------------------------------------
constexpr int kE8Threads = 256;

// sign(x) | E4M3(|x| / s) for one value (s > 0 or s == 0), as the helper of the block scales
// computes it: the reference for the grouped form below and the ragged tail.
__device__ __forceinline__ uint32_t e4m3_tensor_code(float v, float s, float rs)
{
    const uint32_t mag = s > 0.0f ? e4m3_of_quotient(fabsf(v), s, rs) : 0u;
    return mag | ((__float_as_uint(v) >> 24) & 0x80u);
}

// Codes of 8 values (first value in the low byte of .x), s > 0. q = x * RN(1/s) in packed fp32
// multiplies; the hardware pair conversion rounds the signed quotient to nearest (ties to even,
// saturating), which is sign(x) | E4M3(|q|). q is within 3 fp32 ulps of RN(x / s), and the
// E4M3 decision can only differ where q lies within 4 ulps of a midpoint (the 20 mantissa bits
// below the 3 kept ones at 0x80000), in the subnormal E4M3 range, or when q is not finite; if
// any of the 8 values is in such a case, all 8 take the IEEE quotient.
__device__ __forceinline__ uint2 e4m3_codes8(const float (&f)[8], float s, uint64_t rs2)
{
    float q[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint64_t r;
        asm("mul.rn.f32x2 %0, %1, %2;"
            : "=l"(r)
            : "l"(((uint64_t)__float_as_uint(f[2 * j + 1]) << 32) | __float_as_uint(f[2 * j])),
              "l"(rs2));
        q[2 * j] = __uint_as_float((uint32_t)r);
        q[2 * j + 1] = __uint_as_float((uint32_t)(r >> 32));
    }
    bool slow = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float a = fabsf(q[j]);
        const uint32_t mb = __float_as_uint(q[j]) & 0xFFFFFu;
        slow |= (a < 0.015625f && a != 0.0f) || !(a <= 3.0e38f) || (mb - 0x7FFFCu <= 8u);
    }
    if (slow) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            q[j] = __fdiv_rn(f[j], s);
    }
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint16_t h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(q[2 * j + 1]), "f"(q[2 * j]));
        w[j] = h;
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

template <int SRC> __device__ __forceinline__ void load8(const uint8_t *x, int64_t i, float (&f)[8])
{
    if constexpr (SRC == kSrcF32) {
        const uint4 a = __ldcs(reinterpret_cast<const uint4 *>(x + i * 4));
        const uint4 b = __ldcs(reinterpret_cast<const uint4 *>(x + i * 4 + 16));
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j)
            f[j] = __uint_as_float(w[j]);
    } else {
        const uint4 a = __ldcs(reinterpret_cast<const uint4 *>(x + i * 2));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = __uint_as_float(w[j] << 16);
            f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

template <int SRC> __device__ __forceinline__ float value_at(const uint8_t *x, int64_t i)
{
    if constexpr (SRC == kSrcF32)
        return reinterpret_cast<const float *>(x)[i];
    else
        return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(x)[i] << 16);
}

template <int SRC>
__global__ void __launch_bounds__(kE8Threads)
    e4m3_encode_kernel(const uint8_t *__restrict__ x, int64_t n, const float *static_amax,
                       const float *__restrict__ partials, int npartials,
                       uint8_t *__restrict__ codes, float *__restrict__ scale_out)
{
    __shared__ float s_s;
    if (!static_amax)
        pdl_wait(); // the amax kernel's partial maxima are complete and visible
    if (threadIdx.x < 32) {
        float g = 0.0f;
        if (static_amax) {
            g = *static_amax;
        } else {
            for (int i = threadIdx.x; i < npartials; i += 32)
                g = fmaxf(g, __ldcg(partials + i));
            // the amax kernel folds whole 16-byte vectors; the values after the last one
            const int64_t tail0 = ((n * Src<SRC>::kBytes) & ~(int64_t)15) / Src<SRC>::kBytes;
            for (int64_t i = tail0 + threadIdx.x; i < n; i += 32)
                g = fmaxf(g, fabsf(value_at<SRC>(x, i)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
        }
        if (threadIdx.x == 0) {
            const float sc = __fdiv_rn(g, 448.0f);
            s_s = sc;
            if (blockIdx.x == 0)
                *scale_out = sc;
        }
    }
    __syncthreads();
    const float sc = s_s;
    const float rs = __frcp_rn(sc);
    const uint64_t rs2 = ((uint64_t)__float_as_uint(rs) << 32) | __float_as_uint(rs);
    const int64_t nvec = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * kE8Threads;
    for (int64_t v = (int64_t)blockIdx.x * kE8Threads + threadIdx.x; v < nvec; v += stride) {
        float f[8];
        load8<SRC>(x, v * 8, f);
        uint2 c;
        if (sc > 0.0f) {
            c = e4m3_codes8(f, sc, rs2);
        } else { // s == 0: sign-only codes
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j)
                w[j >> 2] |= ((__float_as_uint(f[j]) >> 24) & 0x80u) << (8 * (j & 3));
            c = make_uint2(w[0], w[1]);
        }
        __stcs(reinterpret_cast<uint2 *>(codes + v * 8), c);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n & 7)) { // ragged tail, one value per thread
        const int64_t i = (nvec << 3) + threadIdx.x;
        codes[i] = (uint8_t)e4m3_tensor_code(value_at<SRC>(x, i), sc, rs);
    }
}

// Single-pass FP8 tensorwise quantize for dynamic amax (tensors of 16 MB up to what the CTAs'
// shared memory holds): one CTA per SM bulk-loads its contiguous share of the flat tensor in
// 32 KB copies and folds max |x| as they land, publishes one partial, meets the other CTAs at
// a grid-wide barrier (cooperative launch), reduces the partials to s = amax / 448 and encodes
// from shared memory, 8 values per thread-step (one 8-byte code store; consecutive threads,
// consecutive vectors: conflict-free shared-memory reads and coalesced stores). The tensor is
// read from HBM once and no second kernel runs. n: a multiple of 8.
constexpr int kE8FusedThreads = 1024;

template <int SRC>
__global__ void __launch_bounds__(kE8FusedThreads, 1)
    e4m3_fused_kernel(const uint8_t *__restrict__ x, int64_t n, float *__restrict__ slots,
                      GridBarrier *barrier, uint8_t *__restrict__ codes,
                      float *__restrict__ scale_out, int *status)
{
    extern __shared__ __align__(128) uint8_t buf[];
    pdl_wait(); // programmatic dependent launch: the previous kernel's writes are visible
    __shared__ uint64_t bars[kFusedMaxChunks];
    __shared__ float s_red[kE8FusedThreads / 32];
    __shared__ float s_s;
    constexpr int G = 16 / Src<SRC>::kBytes >= 8 ? 1 : 2; // 16-byte vectors per 8 values
    const int64_t ngroups = n >> 3;
    const int64_t g0 = ngroups * blockIdx.x / gridDim.x;
    const int64_t g1 = ngroups * (blockIdx.x + 1) / gridDim.x;
    const int64_t byte0 = g0 * 16 * G;
    const int64_t nbytes = (g1 - g0) * 16 * G;
    const int nch = (int)((nbytes + kFusedChunk - 1) / kFusedChunk);
    if (threadIdx.x == 0) {
        for (int i = 0; i < nch; ++i)
            mbar_init(&bars[i], 1);
        fence_barrier_init();
        for (int i = 0; i < nch; ++i) {
            const int64_t off = (int64_t)i * kFusedChunk;
            const uint32_t nb = (uint32_t)min((int64_t)kFusedChunk, nbytes - off);
            mbar_arrive_expect_tx(&bars[i], nb);
            bulk_load_1d(buf + off, x + byte0 + off, nb, &bars[i]);
        }
    }
    __syncthreads();
    const uint32_t base = smem_u32(buf);
    uint32_t m = 0;
    for (int c = 0; c < nch; ++c) {
        if (!mbar_wait(&bars[c], 0, kSpinLimit) && (threadIdx.x & 31) == 0)
            atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
        const int nv = (int)(min((int64_t)kFusedChunk, nbytes - (int64_t)c * kFusedChunk) >> 4);
        const uint32_t cb = base + (uint32_t)c * kFusedChunk;
        for (int i = threadIdx.x; i < nv; i += kE8FusedThreads)
            m = mag_fold<SRC>(m, Src<SRC>::vec_magmax(lds128(cb + 16 * i)));
    }
    float f = Src<SRC>::mag_to_f32(m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    if ((threadIdx.x & 31) == 0)
        s_red[threadIdx.x >> 5] = f;
    __syncthreads();
    if (threadIdx.x < 32) {
        float g = s_red[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
        // every CTA's maximum, through the workspace's exchange slots (bounded)
        if (gridDim.x > 1) {
            float unused;
            if (!grid_exchange_max(slots, barrier, (int)gridDim.x, (int)blockIdx.x, g, 0.0f,
                                   kExchangeLimit, g, unused) &&
                threadIdx.x == 0)
                atomicExch(status, (int)NVFP4_ERR_TIMEOUT);
        }
        if (threadIdx.x == 0) {
            const float sc = __fdiv_rn(g, 448.0f);
            s_s = sc;
            if (blockIdx.x == 0)
                *scale_out = sc;
        }
    }
    __syncthreads();
    pdl_launch_dependents(); // a dependent GEMM may set up while this grid encodes
    const float sc = s_s;
    const float rs = __frcp_rn(sc);
    const uint64_t rs2 = ((uint64_t)__float_as_uint(rs) << 32) | __float_as_uint(rs);
    const int ng = (int)(g1 - g0);
    for (int q = threadIdx.x; q < ng; q += kE8FusedThreads) {
        float fv[8];
        if constexpr (SRC == kSrcF32) {
            const uint4 a = lds128(base + 32 * q), b = lds128(base + 32 * q + 16);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j)
                fv[j] = __uint_as_float(w[j]);
        } else {
            const uint4 a = lds128(base + 16 * q);
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                fv[2 * j] = __uint_as_float(w[j] << 16);
                fv[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
        uint2 c;
        if (sc > 0.0f) {
            c = e4m3_codes8(fv, sc, rs2);
        } else { // s == 0: sign-only codes
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j)
                w[j >> 2] |= ((__float_as_uint(fv[j]) >> 24) & 0x80u) << (8 * (j & 3));
            c = make_uint2(w[0], w[1]);
        }
        __stcs(reinterpret_cast<uint2 *>(codes + (g0 + q) * 8), c);
    }
}

template <int SRC>
cudaError_t launch_e4m3_typed(const void *x, int64_t n, const float *static_amax,
                              uint8_t *codes, float *scale_out, void *ws, cudaStream_t s)
{
    const int sms = num_sms();
    int npartials = 0;
    {
        // single pass when every CTA's share fits in its shared memory (16 MB and up, as the
        // NVFP4 fused kernel; n a multiple of 8)
        const int64_t nbytes = n * Src<SRC>::kBytes;
        const int64_t per = ((n >> 3) + sms - 1) / sms * 8 * Src<SRC>::kBytes;
        if (!static_amax && (n & 7) == 0 && nbytes >= kFusedMinBytes && per <= kFusedCap &&
            sms <= kExchangeMaxCtas) {
            static std::once_flag fattr[64];
            static cudaError_t fe[64];
            int dev = 0;
            cudaGetDevice(&dev);
            std::call_once(fattr[dev & 63], [&]() {
                fe[dev & 63] = cudaFuncSetAttribute(
                    e4m3_fused_kernel<SRC>, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedCap);
            });
            if (fe[dev & 63] != cudaSuccess)
                return fe[dev & 63];
            GridBarrier *bar = grid_barrier_for(s);
            if (!bar)
                return cudaErrorInvalidValue;
            cudaLaunchConfig_t fc{};
            fc.gridDim = dim3((unsigned)sms);
            fc.blockDim = dim3(kE8FusedThreads);
            fc.dynamicSmemBytes = kFusedCap;
            fc.stream = s;
            cudaLaunchAttribute fa[2];
            fa[0].id = cudaLaunchAttributeCooperative;
            fa[0].val.cooperative = 1;
            fa[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            fa[1].val.programmaticStreamSerializationAllowed = 1;
            fc.attrs = fa;
            fc.numAttrs = 2;
            return cudaLaunchKernelEx(&fc, e4m3_fused_kernel<SRC>,
                                      reinterpret_cast<const uint8_t *>(x), n,
                                      reinterpret_cast<float *>(ws), bar, codes, scale_out,
                                      device_status_ptr());
        }
    }
    if (!static_amax) {
        const int64_t nbytes = n * Src<SRC>::kBytes;
        int g = sms < kAmaxPartials ? sms : kAmaxPartials;
        const int64_t need = (nbytes + kChunk - 1) / kChunk;
        if (need < g)
            g = need < 1 ? 1 : (int)need;
        npartials = g;
        const size_t smem = (size_t)kRing * kChunk;
        cudaError_t e = cudaFuncSetAttribute(amax_kernel<SRC>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        amax_kernel<SRC><<<g, kAmaxThreads, smem, s>>>(reinterpret_cast<const uint8_t *>(x),
                                                       nbytes, reinterpret_cast<float *>(ws),
                                                       device_status_ptr());
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    const int64_t nvec = n >> 3;
    int64_t grid = (nvec + kE8Threads - 1) / kE8Threads;
    const int64_t max_grid = (int64_t)sms * 8;
    if (grid > max_grid)
        grid = max_grid;
    if (grid < 1)
        grid = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kE8Threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = static_amax ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, e4m3_encode_kernel<SRC>, reinterpret_cast<const uint8_t *>(x),
                              n, static_amax, reinterpret_cast<const float *>(ws), npartials, codes,
                              scale_out);
}

} // namespace

size_t quantize_workspace_bytes() { return (size_t)kAmaxPartials * sizeof(float); }

cudaError_t launch_quantize(const void *x, int src_type, const float *fp8_scale, int64_t rows,
                            int64_t cols, const float *static_amax, uint8_t *codes,
                            uint8_t *scales_swz, uint8_t *scales_lin, float *global_scale,
                            void *ws, cudaStream_t s)
{
    switch (src_type) {
    case kSrcF32:
        return launch_typed<kSrcF32>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                     scales_lin, global_scale, ws, s);
    case kSrcBF16:
        return launch_typed<kSrcBF16>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                      scales_lin, global_scale, ws, s);
    default:
        return launch_typed<kSrcE4M3>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                      scales_lin, global_scale, ws, s);
    }
}

cudaError_t launch_quantize_e4m3(const void *x, int src_type, int64_t n, const float *static_amax,
                                 uint8_t *codes, float *scale_out, void *ws, cudaStream_t s)
{
    if (src_type == kSrcF32)
        return launch_e4m3_typed<kSrcF32>(x, n, static_amax, codes, scale_out, ws, s);
    return launch_e4m3_typed<kSrcBF16>(x, n, static_amax, codes, scale_out, ws, s);
}

// Two tensors in one cooperative launch (fused_pair_quantize_kernel): a, the larger, held in
// shared memory, b in registers. Taken when a's share per SM fits at kPairThreads, b's share
// fits the threads' registers (about 9.7 MB of fp8, bf16 or fp32 on 148 SMs) and
// the pair is large enough for the single pass to pay (16 MB, the single-tensor fused
// kernel's floor). Returns false when the pair does not qualify (nothing launched).
template <int SA, int SB>
cudaError_t launch_fused_pair_typed(const QuantArgs &a, const QuantArgs &b, int grid, bool coop,
                                    cudaStream_t s)
{
    constexpr int kSmem = kFusedCap;
    static std::once_flag fattr[64];
    static cudaError_t fe[64];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(fattr[dev & 63], [&]() {
        fe[dev & 63] = cudaFuncSetAttribute(fused_pair_quantize_kernel<SA, SB>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    });
    if (fe[dev & 63] != cudaSuccess)
        return fe[dev & 63];
    cudaLaunchConfig_t fc{};
    fc.gridDim = dim3((unsigned)grid);
    fc.blockDim = dim3(kPairThreads);
    fc.dynamicSmemBytes = kSmem;
    fc.stream = s;
    cudaLaunchAttribute fa[2];
    fa[0].id = cudaLaunchAttributeCooperative;
    fa[0].val.cooperative = coop ? 1 : 0;
    fa[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    fa[1].val.programmaticStreamSerializationAllowed = 1;
    fc.attrs = fa;
    fc.numAttrs = 2;
    return cudaLaunchKernelEx(&fc, fused_pair_quantize_kernel<SA, SB>, a, b);
}

template <int SA>
cudaError_t launch_fused_pair_b(int sb, const QuantArgs &a, const QuantArgs &b, int grid,
                                bool coop, cudaStream_t s)
{
    switch (sb) {
    case kSrcF32: return launch_fused_pair_typed<SA, kSrcF32>(a, b, grid, coop, s);
    case kSrcBF16: return launch_fused_pair_typed<SA, kSrcBF16>(a, b, grid, coop, s);
    default: return launch_fused_pair_typed<SA, kSrcE4M3>(a, b, grid, coop, s);
    }
}

int64_t enc_item_bytes(int src) { return src == kSrcF32 ? 2048 : src == kSrcBF16 ? 2048 : 1024; }

bool try_fused_pair(const QuantGroup &g, void *ws, cudaStream_t s, cudaError_t *err)
{
    if (g.njobs != 2)
        return false;
    const int ia = g.job[0].nbytes >= g.job[1].nbytes ? 0 : 1, ib = 1 - ia;
    QuantArgs a = g.job[ia], b = g.job[ib];
    const int grid = num_sms();
    // b must fit in registers: kPairRegVecs 16-byte vectors a thread (whole blocks of it)
    const int64_t b_blocks = (int64_t)b.rows * (b.cols / 16);
    const int64_t b_bpt = kPairRegVecs / (g.src[ib] == kSrcF32 ? 4 : g.src[ib] == kSrcBF16 ? 2 : 1);
    if (grid > kExchangeMaxCtas || a.nbytes + b.nbytes < kFusedMinBytes ||
        b.nbytes <= 0 || b_blocks > (int64_t)grid * kPairThreads * b_bpt)
        return false;
    // warp items of a (Enc<>: 32 blocks of fp32, 64 of bf16 / fp8; 2 KB / 2 KB / 1 KB)
    const int64_t item_blocks = g.src[ia] == kSrcF32 ? 32 : 64;
    const int64_t item = enc_item_bytes(g.src[ia]);
    const int64_t nitems = ((int64_t)a.rows * (a.cols / 16) + item_blocks - 1) / item_blocks;
    const int64_t items_per_warp_max = kFusedCap / item / (kPairThreads / 32);
    if ((nitems + grid - 1) / grid > items_per_warp_max * (kPairThreads / 32))
        return false;
    const bool coop = !a.static_amax || !b.static_amax;
    a.slots = b.slots = reinterpret_cast<float *>(ws); // one slot per CTA for both tensors
    a.barrier = b.barrier = coop ? grid_barrier_for(s) : nullptr;
    if (coop && !a.barrier) {
        *err = cudaErrorInvalidValue;
        return true;
    }
    switch (g.src[ia]) {
    case kSrcF32: *err = launch_fused_pair_b<kSrcF32>(g.src[ib], a, b, grid, coop, s); break;
    case kSrcBF16: *err = launch_fused_pair_b<kSrcBF16>(g.src[ib], a, b, grid, coop, s); break;
    default: *err = launch_fused_pair_b<kSrcE4M3>(g.src[ib], a, b, grid, coop, s); break;
    }
    return true;
}

cudaError_t launch_quantize_batch(const QuantJob *jobs, int njobs, void *ws, cudaStream_t s)
{
    const int sms = num_sms();
    QuantGroup g{};
    g.njobs = njobs;
    int64_t amax_w[kMaxQuantJobs], amax_cap[kMaxQuantJobs], enc_w[kMaxQuantJobs],
        enc_cap[kMaxQuantJobs];
    bool dynamic = false;
    for (int j = 0; j < njobs; ++j) {
        const QuantJob &jb = jobs[j];
        g.src[j] = jb.src;
        switch (jb.src) {
        case kSrcF32: fill_args<kSrcF32>(g.job[j], jb); break;
        case kSrcBF16: fill_args<kSrcBF16>(g.job[j], jb); break;
        default: fill_args<kSrcE4M3>(g.job[j], jb); break;
        }
        const int64_t nbytes = g.job[j].nbytes;
        const bool dyn = !jb.static_amax && nbytes > 0;
        dynamic = dynamic || dyn;
        amax_w[j] = dyn ? nbytes : 0;
        amax_cap[j] = (nbytes + kChunk - 1) / kChunk;
        enc_w[j] = nbytes > 0 ? nbytes : 0;
        enc_cap[j] = jb.rows;
    }
    {
        cudaError_t fe = cudaSuccess;
        if (try_fused_pair(g, ws, s, &fe))
            return fe;
    }
    int amax_total = sms < kAmaxPartials ? sms : kAmaxPartials;
    const int na = split_ctas(njobs, amax_w, amax_cap, amax_total, g.amax_cta0);
    for (int j = 0; j < njobs; ++j) {
        g.job[j].partials = reinterpret_cast<const float *>(ws) + g.amax_cta0[j];
        g.job[j].npartials = g.amax_cta0[j + 1] - g.amax_cta0[j];
    }
    const int ne = split_ctas(njobs, enc_w, enc_cap, sms, g.enc_cta0);
    cudaError_t e;
    if (dynamic && na > 0) {
        const size_t smem = (size_t)kRing * kChunk;
        static std::once_flag attr[64];
        int dev = 0;
        cudaGetDevice(&dev);
        cudaError_t ae = cudaSuccess;
        std::call_once(attr[dev & 63], [&]() {
            ae = cudaFuncSetAttribute(amax_group_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        });
        if (ae != cudaSuccess)
            return ae;
        amax_group_kernel<<<na, kAmaxThreads, smem, s>>>(g);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    if (ne == 0)
        return cudaSuccess;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ne);
    cfg.blockDim = dim3(kEncThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = (dynamic && na > 0) ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_group_kernel, g);
}

} // namespace nvfp4
