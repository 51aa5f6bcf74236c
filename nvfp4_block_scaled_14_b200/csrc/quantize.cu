// quantize.cu -- NVFP4 quantization of fp32 / bf16 / FP8-E4M3 tensors on sm_100a.
//
// Format and decode rule: "Qwen-Image NVFP4 on a 16 GB Ada GPU", section "What NVFP4 is and
// how it differs from NF4" (E2M1 codes, one FP8 scale per 16 values, one FP32 global scale)
// and the figure "First NVFP4 block, as stored in the file" (low nibble first,
// weight = E2M1 x block scale x global scale). Dynamic per-tensor amax for activations:
// "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details". FP8 source (double
// quantization): "Qwen-Rapid-AIO FP8 -> NVFP4", "1. Double Quantization".
//
// Two kernels, both HBM-bound:
//   amax_kernel   -- grid-stride max |x| with 128-bit loads; one partial per CTA (no atomics,
//                    no zeroing, order-free and therefore exact).
//   encode_kernel -- one CTA per 128-row x 64-column tile (exactly one 512-byte atom of the
//                    tensor-core scale layout); each thread encodes two 16-value blocks:
//                    block amax, E4M3 scale, reciprocal, E2M1 codes by the hardware cvt,
//                    8-byte code stores (four lanes write 32 contiguous bytes of a row) and
//                    byte stores of the swizzled and / or linear scales. Padding entries of
//                    the swizzled atom are written as zero by the same CTA.
// Code-deciding arithmetic is IEEE fp32 round-to-nearest in a fixed order (__fdiv_rn,
// __fmul_rn, __frcp_rn): sg = amax / 2688, sb = E4M3(bmax / (sg * 6)),
// code = E2M1(x * (1 / (sb * sg))).
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kAmaxThreads = 512;
constexpr int kEncThreads = 256;

template <int SRC> struct Src;

template <> struct Src<kSrcF32> {
    static constexpr int kBytes = 4;
    __device__ static float vec_absmax(uint4 v)
    {
        float a = fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y)));
        float b = fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)));
        return fmaxf(a, b);
    }
};

template <> struct Src<kSrcBF16> {
    static constexpr int kBytes = 2;
    __device__ static float vec_absmax(uint4 v)
    {
        // |x| of a bf16 is monotone in its low 15 bits: take the max of the magnitude bits.
        uint32_t m = 0;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m = max(m, w[i] & 0x7FFFu);
            m = max(m, (w[i] >> 16) & 0x7FFFu);
        }
        return __uint_as_float(m << 16);
    }
};

template <> struct Src<kSrcE4M3> {
    static constexpr int kBytes = 1;
    __device__ static float vec_absmax(uint4 v)
    {
        // |e4m3| is monotone in its low 7 bits (finite inputs).
        uint32_t m = 0;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int b = 0; b < 4; ++b)
                m = max(m, (w[i] >> (8 * b)) & 0x7Fu);
        return e4m3_to_f32(m);
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

template <int SRC>
__global__ void __launch_bounds__(kAmaxThreads)
    amax_kernel(const uint4 *__restrict__ x, int64_t nvec, float *__restrict__ partials)
{
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * kAmaxThreads;
    int64_t i = (int64_t)blockIdx.x * kAmaxThreads + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 v0 = ldg_stream(x + i), v1 = ldg_stream(x + i + stride);
        uint4 v2 = ldg_stream(x + i + 2 * stride), v3 = ldg_stream(x + i + 3 * stride);
        m = fmaxf(m, fmaxf(fmaxf(Src<SRC>::vec_absmax(v0), Src<SRC>::vec_absmax(v1)),
                           fmaxf(Src<SRC>::vec_absmax(v2), Src<SRC>::vec_absmax(v3))));
    }
    for (; i < nvec; i += stride)
        m = fmaxf(m, Src<SRC>::vec_absmax(ldg_stream(x + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float red[kAmaxThreads / 32];
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (threadIdx.x == 0)
            partials[blockIdx.x] = m;
    }
}

// Load one 16-value block as fp32 (fp8: upcast by one fp32 multiply with s8).
template <int SRC>
__device__ __forceinline__ void load_block(const uint8_t *p, float s8, float (&v)[16])
{
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
    if constexpr (SRC == kSrcF32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 w = ldg_stream(q + i);
            v[4 * i + 0] = __uint_as_float(w.x);
            v[4 * i + 1] = __uint_as_float(w.y);
            v[4 * i + 2] = __uint_as_float(w.z);
            v[4 * i + 3] = __uint_as_float(w.w);
        }
    } else if constexpr (SRC == kSrcBF16) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 w = ldg_stream(q + i);
            uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j + 0] = __uint_as_float(u[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
        }
    } else {
        uint4 w = ldg_stream(q);
        uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 a = e4m3x2_to_f32x2(u[j] & 0xFFFFu);
            float2 b = e4m3x2_to_f32x2(u[j] >> 16);
            v[4 * j + 0] = __fmul_rn(a.x, s8);
            v[4 * j + 1] = __fmul_rn(a.y, s8);
            v[4 * j + 2] = __fmul_rn(b.x, s8);
            v[4 * j + 3] = __fmul_rn(b.y, s8);
        }
    }
}

// Encode one block: returns the E4M3 scale byte and writes the 8 code bytes.
__device__ __forceinline__ uint32_t encode_block(const float (&v)[16], float sg, float t,
                                                 uint2 &packed)
{
    float bmax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        bmax = fmaxf(bmax, fabsf(v[j]));
    uint32_t sb = 0;
    if (sg > 0.0f)
        sb = cvt_e4m3(__fdiv_rn(bmax, t));
    const float fsb = e4m3_to_f32(sb);
    packed = make_uint2(0u, 0u);
    if (fsb != 0.0f) {
        const float rcp = __frcp_rn(__fmul_rn(fsb, sg));
        float y[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            y[j] = __fmul_rn(v[j], rcp);
        packed.x = cvt_e2m1x8(y);
        packed.y = cvt_e2m1x8(y + 8);
    }
    return sb;
}

template <int SRC>
__global__ void __launch_bounds__(kEncThreads)
    encode_kernel(const uint8_t *__restrict__ x, const float *__restrict__ fp8_scale,
                  int64_t rows, int64_t cols, const float *__restrict__ static_amax,
                  const float *__restrict__ partials, int npartials, uint8_t *__restrict__ codes,
                  uint8_t *__restrict__ sf_swz, uint8_t *__restrict__ sf_lin,
                  float *__restrict__ global_scale)
{
    __shared__ float s_sg;
    const float s8 = (SRC == kSrcE4M3 && fp8_scale) ? *fp8_scale : 1.0f;
    if (threadIdx.x < 32) {
        float a = 0.0f;
        if (static_amax) {
            a = *static_amax;
        } else {
            for (int i = threadIdx.x; i < npartials; i += 32)
                a = fmaxf(a, partials[i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            if (SRC == kSrcE4M3)
                a = __fmul_rn(a, s8); // max |e| * s8 == max |e * s8| (rounding is monotone)
        }
        if (threadIdx.x == 0) {
            const float sg = __fdiv_rn(a, 2688.0f); // 6 * 448
            s_sg = sg;
            if (blockIdx.x == 0)
                *global_scale = sg;
        }
    }
    __syncthreads();
    const float sg = s_sg;
    const float t = __fmul_rn(sg, 6.0f);

    const int64_t nb = cols >> 4;
    const int64_t apb = (nb + 3) >> 2; // atoms per 128-row band
    const int64_t ntiles = ((rows + 127) >> 7) * apb;
    const int64_t row_bytes = cols * Src<SRC>::kBytes;

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t band = tile / apb, atom = tile - band * apb;
        float v[2][16];
        int64_t row[2], blk[2];
        bool valid[2];
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int local = threadIdx.x + it * kEncThreads; // 0..511
            row[it] = band * 128 + (local >> 2);
            blk[it] = atom * 4 + (local & 3);
            valid[it] = row[it] < rows && blk[it] < nb;
            if (valid[it])
                load_block<SRC>(x + row[it] * row_bytes + blk[it] * 16 * Src<SRC>::kBytes, s8,
                                v[it]);
        }
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            uint32_t sb = 0;
            if (valid[it]) {
                uint2 packed;
                sb = encode_block(v[it], sg, t, packed);
                *reinterpret_cast<uint2 *>(codes + row[it] * (cols >> 1) + blk[it] * 8) = packed;
                if (sf_lin)
                    sf_lin[row[it] * nb + blk[it]] = (uint8_t)sb;
            }
            if (sf_swz) {
                const int local = threadIdx.x + it * kEncThreads;
                const int r = local >> 2;
                sf_swz[tile * 512 + ((r & 31) << 4) + ((r >> 5) << 2) + (local & 3)] =
                    (uint8_t)sb;
            }
        }
    }
}

template <int SRC>
cudaError_t launch_typed(const void *x, const float *fp8_scale, int64_t rows, int64_t cols,
                         const float *static_amax, uint8_t *codes, uint8_t *sf_swz,
                         uint8_t *sf_lin, float *global_scale, float *partials, cudaStream_t s)
{
    int npartials = 0;
    if (!static_amax) {
        const int64_t nvec = rows * cols * Src<SRC>::kBytes / 16;
        int64_t g = (nvec + kAmaxThreads * 4 - 1) / (kAmaxThreads * 4);
        g = g < 1 ? 1 : (g > kAmaxPartials ? kAmaxPartials : g);
        npartials = (int)g;
        amax_kernel<SRC><<<(unsigned)g, kAmaxThreads, 0, s>>>(
            reinterpret_cast<const uint4 *>(x), nvec, partials);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    const int64_t nb = cols >> 4;
    const int64_t ntiles = ((rows + 127) >> 7) * ((nb + 3) >> 2);
    int64_t g = ntiles < 1 ? 1 : ntiles;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap)
        g = cap;
    encode_kernel<SRC><<<(unsigned)g, kEncThreads, 0, s>>>(
        reinterpret_cast<const uint8_t *>(x), fp8_scale, rows, cols, static_amax, partials,
        npartials, codes, sf_swz, sf_lin, global_scale);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_quantize(const void *x, int src_type, const float *fp8_scale, int64_t rows,
                            int64_t cols, const float *static_amax, uint8_t *codes,
                            uint8_t *scales_swz, uint8_t *scales_lin, float *global_scale,
                            float *ws_partials, cudaStream_t s)
{
    switch (src_type) {
    case kSrcF32:
        return launch_typed<kSrcF32>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                     scales_lin, global_scale, ws_partials, s);
    case kSrcBF16:
        return launch_typed<kSrcBF16>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                      scales_lin, global_scale, ws_partials, s);
    default:
        return launch_typed<kSrcE4M3>(x, fp8_scale, rows, cols, static_amax, codes, scales_swz,
                                      scales_lin, global_scale, ws_partials, s);
    }
}

} // namespace nvfp4
