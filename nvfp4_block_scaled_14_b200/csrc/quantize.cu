// quantize.cu -- NVFP4 quantization of fp32 / bf16 / FP8-E4M3 tensors on sm_100a.
//
// Format and decode rule: "Qwen-Image NVFP4 on a 16 GB Ada GPU", section "What NVFP4 is and
// how it differs from NF4" (E2M1 codes, one FP8 scale per 16 values, one FP32 global scale)
// and the figure "First NVFP4 block, as stored in the file" (low nibble first,
// weight = E2M1 x block scale x global scale). Dynamic per-tensor amax for activations:
// "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details". FP8 source (double
// quantization): "Qwen-Rapid-AIO FP8 -> NVFP4", "1. Double Quantization".
//
// Two kernels per call, both HBM-bound, chained by programmatic dependent launch:
//   amax_kernel   (dynamic amax only) -- one CTA per SM streams a contiguous byte range of
//                 the tensor through a 4 x 32 KB shared-memory ring of 1-D bulk copies and
//                 reduces max |x| with SIMD integer max on the magnitude bits (exact,
//                 order-free); one partial per CTA, no atomics, nothing to zero.
//   encode_kernel -- one CTA per SM owns a contiguous range of rows; each warp takes a
//                 64-block run of one row (1024 values, fully coalesced), two 16-value blocks per
//                 lane. It loads its first items before griddepcontrol.wait, so the loads
//                 overlap the amax kernel's tail (the tensor is then mostly in L2), reduces the
//                 partial maxima to the global scale, and fills a 128-entry table of
//                 1 / (E4M3(c) * sg). Per block: block amax, E4M3 scale, E2M1 codes by the
//                 hardware cvt, a 16-byte code store (a warp writes 512 contiguous bytes) and
//                 16-bit stores of the swizzled and / or linear scales; atom padding is zeroed.
// Code-deciding arithmetic is IEEE fp32 round-to-nearest in a fixed order (__fdiv_rn,
// __fmul_rn, __frcp_rn): sg = amax / 2688, sb = E4M3(bmax / (sg * 6)),
// code = E2M1(x * (1 / (sb * sg))).
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 1024;      // encode: 32 warps, one 16-value block per lane per item
constexpr int kAmaxThreads = 1024;  // amax: one CTA per SM streaming its byte range
constexpr int kChunk = 32 * 1024;   // amax ring: 4 x 32 KB bulk copies in flight per SM
constexpr int kRing = 4;
constexpr uint32_t kSpinLimit = 1u << 24;

template <int SRC> struct Src;

// |x| orders like the magnitude bits of x for finite values, so maxima are taken on the bit
// patterns with SIMD integer max: exact, order-free.
template <> struct Src<kSrcF32> {
    static constexpr int kBytes = 4;
    __device__ static uint32_t vec_magmax(uint4 v) // fp32 magnitude bits
    {
        return max(max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu),
                   max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu));
    }
    __device__ static float mag_to_f32(uint32_t m) { return __uint_as_float(m); }
};

template <> struct Src<kSrcBF16> {
    static constexpr int kBytes = 2;
    __device__ static uint32_t vec_magmax(uint4 v) // two 16-bit lanes of magnitude bits
    {
        const uint32_t k = 0x7FFF7FFFu;
        return __vmaxu2(__vmaxu2(v.x & k, v.y & k), __vmaxu2(v.z & k, v.w & k));
    }
    __device__ static float mag_to_f32(uint32_t m)
    {
        return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
    }
};

template <> struct Src<kSrcE4M3> {
    static constexpr int kBytes = 1;
    __device__ static uint32_t vec_magmax(uint4 v) // four 8-bit lanes of magnitude bits
    {
        const uint32_t k = 0x7F7F7F7Fu;
        return __vmaxu4(__vmaxu4(v.x & k, v.y & k), __vmaxu4(v.z & k, v.w & k));
    }
    __device__ static float mag_to_f32(uint32_t m) // |e4m3| (before the fp8 scale)
    {
        const uint32_t b = max(max(m & 0xFFu, (m >> 8) & 0xFFu),
                               max((m >> 16) & 0xFFu, m >> 24));
        return e4m3_to_f32(b);
    }
};

__device__ __forceinline__ uint4 ldg_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Raw 16-byte vectors of one 16-value block: 4 (fp32), 2 (bf16) or 1 (fp8).
template <int SRC> constexpr int kVecs = SRC == kSrcF32 ? 4 : (SRC == kSrcBF16 ? 2 : 1);

template <int SRC>
__device__ __forceinline__ void load_raw(const uint8_t *p, uint4 (&r)[4])
{
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < kVecs<SRC>; ++i)
        r[i] = ldg_stream(q + i);
}

// Raw block -> 16 fp32 values (bf16 widening is exact; fp8 is upcast by one fp32 multiply
// with s8).
template <int SRC>
__device__ __forceinline__ void to_f32(const uint4 (&r)[4], float s8, float (&v)[16])
{
    if constexpr (SRC == kSrcF32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i + 0] = __uint_as_float(r[i].x);
            v[4 * i + 1] = __uint_as_float(r[i].y);
            v[4 * i + 2] = __uint_as_float(r[i].z);
            v[4 * i + 3] = __uint_as_float(r[i].w);
        }
    } else if constexpr (SRC == kSrcBF16) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t u[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j + 0] = __uint_as_float(u[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
        }
    } else {
        const uint32_t u[4] = {r[0].x, r[0].y, r[0].z, r[0].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 ss = make_float2(s8, s8);
            const float2 a = __fmul2_rn(e4m3x2_to_f32x2(u[j] & 0xFFFFu), ss);
            const float2 b = __fmul2_rn(e4m3x2_to_f32x2(u[j] >> 16), ss);
            v[4 * j + 0] = a.x;
            v[4 * j + 1] = a.y;
            v[4 * j + 2] = b.x;
            v[4 * j + 3] = b.y;
        }
    }
}

// Block maximum |x| (fp32) from the raw vectors (fp8: times s8, which commutes with the max
// because rounding is monotone).
template <int SRC>
__device__ __forceinline__ float block_absmax(const uint4 (&r)[4], float s8)
{
    if constexpr (SRC == kSrcF32) {
        return __uint_as_float(max(max(Src<SRC>::vec_magmax(r[0]), Src<SRC>::vec_magmax(r[1])),
                                   max(Src<SRC>::vec_magmax(r[2]), Src<SRC>::vec_magmax(r[3]))));
    } else if constexpr (SRC == kSrcBF16) {
        return Src<SRC>::mag_to_f32(
            __vmaxu2(Src<SRC>::vec_magmax(r[0]), Src<SRC>::vec_magmax(r[1])));
    } else {
        return __fmul_rn(Src<SRC>::mag_to_f32(Src<SRC>::vec_magmax(r[0])), s8);
    }
}

// E4M3 code of RN(bmax / t), exactly as cvt_e4m3(__fdiv_rn(bmax, t)) gives it, usually without
// the division. rt = RN(1/t). q0 = RN(bmax * rt) is within 3 fp32 ulps of RN(bmax / t) (two
// roundings of relative size 2^-24 each, plus the rounding of the quotient itself). For
// q0 >= 2^-6 (normal E4M3 range) the E4M3 rounding decision depends on the 20 fp32 mantissa
// bits below the 3 kept ones and flips only at 0x80000 (the midpoint between two E4M3
// values; saturation at 448 leaves no further boundary above). If q0 sits more than 4 ulps
// from that midpoint, q0 and RN(bmax / t) round to the same E4M3 code; otherwise, below
// 2^-6, and when q0 is not finite (1/t overflowed), the correctly rounded division decides.
__device__ __forceinline__ uint32_t e4m3_of_quotient(float bmax, float t, float rt)
{
    if (bmax == 0.0f)
        return 0u;
    const float q0 = __fmul_rn(bmax, rt);
    const int d = (int)(__float_as_uint(q0) & 0xFFFFFu) - 0x80000;
    if (q0 >= 0.015625f && q0 <= 3.0e38f && (d > 4 || d < -4))
        return cvt_e4m3(q0);
    return cvt_e4m3(__fdiv_rn(bmax, t));
}

// Encode one block: returns the E4M3 scale byte and writes the 8 code bytes. rcp_tab[c] holds
// 1 / (E4M3(c) * sg), computed with the same two round-to-nearest operations per code.
template <int SRC>
__device__ __forceinline__ uint32_t encode_block(const uint4 (&r)[4], float s8, float sg,
                                                 float t, float rt, const float *rcp_tab,
                                                 uint2 &packed)
{
    const float bmax = block_absmax<SRC>(r, s8);
    uint32_t sb = 0;
    if (sg > 0.0f)
        sb = e4m3_of_quotient(bmax, t, rt);
    packed = make_uint2(0u, 0u);
    if (sb != 0u) {
        float v[16];
        to_f32<SRC>(r, s8, v);
        const float rcp = rcp_tab[sb];
        const float2 rr = make_float2(rcp, rcp);
        float y[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            const float2 p = __fmul2_rn(make_float2(v[j], v[j + 1]), rr);
            y[j] = p.x;
            y[j + 1] = p.y;
        }
        packed.x = cvt_e2m1x8(y);
        packed.y = cvt_e2m1x8(y + 8);
    }
    return sb;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Fold a magnitude-bit accumulator (per source type) into another.
template <int SRC> __device__ __forceinline__ uint32_t mag_fold(uint32_t a, uint32_t b)
{
    if constexpr (SRC == kSrcF32)
        return max(a, b);
    else if constexpr (SRC == kSrcBF16)
        return __vmaxu2(a, b);
    else
        return __vmaxu4(a, b);
}

template <int SRC> __device__ __forceinline__ uint32_t raw_magmax(const uint4 (&r)[4])
{
    uint32_t m = Src<SRC>::vec_magmax(r[0]);
#pragma unroll
    for (int i = 1; i < kVecs<SRC>; ++i)
        m = mag_fold<SRC>(m, Src<SRC>::vec_magmax(r[i]));
    return m;
}

struct QuantArgs {
    const uint8_t *x;
    const float *fp8_scale;
    int rows, cols;
    const float *static_amax;
    uint8_t *codes, *sf_swz, *sf_lin;
    float *global_scale;
    const float *partials; // one max |x| per amax CTA (dynamic amax)
    int npartials;
    uint32_t chunks_magic; // ceil(2^32 / runs) for runs >= 2: item / runs by umulhi
};

// K1: max |x| over a contiguous byte range per CTA, streamed through a shared-memory ring
// with 1-D bulk copies; one partial per CTA.
template <int SRC>
__global__ void __launch_bounds__(kAmaxThreads, 1)
    amax_kernel(const uint8_t *__restrict__ x, int64_t nbytes, float *__restrict__ partials,
                int *status)
{
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t bars[kRing];
    __shared__ float s_red[kAmaxThreads / 32];
    const int64_t nvec = nbytes >> 4;
    const int64_t per = ((nvec + gridDim.x - 1) / gridDim.x) << 4;
    const int64_t b0 = min(nbytes, per * (int64_t)blockIdx.x);
    const int64_t b1 = min(nbytes, b0 + per);
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
            partials[blockIdx.x] = f;
    }
}

// K2: encode. Each CTA owns a contiguous range of rows; each warp takes a 64-block run of one
// row and each lane two adjacent 16-value blocks, so address arithmetic and loop control are
// shared by two blocks, the codes leave as one 16-byte store and the two scale bytes as one
// 16-bit store. The first item is loaded before waiting on the amax kernel (programmatic
// dependent launch), so the loads overlap its tail; later items are double-buffered.
template <int SRC>
__global__ void __launch_bounds__(kThreads, 1) encode_kernel(const QuantArgs a)
{
    __shared__ float s_sg;
    __shared__ float s_rcp[128];
    constexpr int kBlkBytes = 16 * Src<SRC>::kBytes;
    constexpr int V = kVecs<SRC>; // 16-byte vectors per block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = a.cols >> 4;       // blocks per row
    const int runs = (nb + 63) >> 6;  // 64-block runs per row (one per warp item)
    const int apb = (nb + 3) >> 2;    // scale atoms per 128-row band
    const int64_t row_bytes = (int64_t)a.cols * Src<SRC>::kBytes;
    const int r0 = (int)((int64_t)a.rows * blockIdx.x / gridDim.x);
    const int r1 = (int)((int64_t)a.rows * (blockIdx.x + 1) / gridDim.x);
    const int items = (r1 - r0) * runs;
    const uint8_t *xbase = a.x + (int64_t)r0 * row_bytes;

    // item -> (row offset, first block of this lane). The quotient by multiply-high is exact
    // or one too large (item < 2^31, runs < 2^26); one correction.
    auto item_rb = [&](int it, int &ro, int &b0) {
        if (runs == 1) {
            ro = it;
            b0 = 2 * lane;
            return;
        }
        ro = (int)__umulhi((uint32_t)it, a.chunks_magic);
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
            for (int i = threadIdx.x; i < a.npartials; i += 32)
                g = fmaxf(g, __ldcg(a.partials + i));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                g = fmaxf(g, __shfl_xor_sync(0xFFFFFFFFu, g, o));
            if (SRC == kSrcE4M3)
                g = __fmul_rn(g, s8); // max |e| * s8 == max |e * s8| (rounding is monotone)
        }
        if (threadIdx.x == 0) {
            const float sg = __fdiv_rn(g, 2688.0f); // 6 * 448
            s_sg = sg;
            if (blockIdx.x == 0)
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

    // blocks b0, b0 + 1 of row r0 + ro: codes, scales; atom padding blocks get zero scales
    auto encode_store = [&](int ro, int b0, const uint4 (&r)[8]) {
        const int row = r0 + ro;
        uint32_t sb0 = 0, sb1 = 0;
        uint2 p0 = make_uint2(0u, 0u), p1 = make_uint2(0u, 0u);
        if (b0 < nb) {
            uint4 x0[4], x1[4];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                x0[v] = r[v];
                x1[v] = r[V + v];
            }
            sb0 = encode_block<SRC>(x0, s8, sg, t, rt, s_rcp, p0);
            uint8_t *c = a.codes + (int64_t)row * (a.cols >> 1) + b0 * 8;
            if (b0 + 1 < nb) {
                sb1 = encode_block<SRC>(x1, s8, sg, t, rt, s_rcp, p1);
                *reinterpret_cast<uint4 *>(c) = make_uint4(p0.x, p0.y, p1.x, p1.y);
            } else {
                *reinterpret_cast<uint2 *>(c) = p0;
            }
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
            it += 32;
            load_item(it, ra, roa, b0a);
        }
    } else {
        while (it < items) {
            load_item(it + 32, rb, rob, b0b);
            encode_store(roa, b0a, ra);
            it += 32;
            if (it >= items)
                break;
            load_item(it + 32, ra, roa, b0a);
            encode_store(rob, b0b, rb);
            it += 32;
        }
    }
    // zero the scale padding rows of the last 128-row band
    if (a.sf_swz) {
        const int rows_pad = ((a.rows + 127) >> 7) << 7;
        for (int row = a.rows + blockIdx.x; row < rows_pad; row += gridDim.x)
            for (int b = threadIdx.x; b < 4 * apb; b += kThreads)
                a.sf_swz[((int64_t)(row >> 7) * apb + (b >> 2)) * 512 + ((row & 31) << 4) +
                         (((row >> 5) & 3) << 2) + (b & 3)] = 0;
    }
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
    const uint64_t runs = (uint64_t)((cols / 16 + 63) / 64);
    qa.chunks_magic = runs > 1 ? (uint32_t)((((uint64_t)1 << 32) + runs - 1) / runs) : 0u;
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
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = static_amax ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_kernel<SRC>, qa);
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

} // namespace nvfp4
