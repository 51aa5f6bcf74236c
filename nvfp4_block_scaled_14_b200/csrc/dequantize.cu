// dequantize.cu -- NVFP4 -> fp32 / bf16 on sm_100a.
//
// weight = E2M1 x block scale x global scale ("Qwen-Image NVFP4 on a 16 GB Ada GPU", worked
// example under the figure "First NVFP4 block, as stored in the file"), computed as
// (E2M1 * sb) * sg with two fp32 round-to-nearest multiplies; bf16 output rounds that value
// to nearest even. The page's own Ada expander does the same job with a 256-entry byte
// table in PyTorch ("Running the NVFP4 weights on Ada"); here the hardware cvt decodes two
// codes at a time.
//
// One thread per 16-value block: an 8-byte code load (a warp reads 256 contiguous bytes),
// one scale byte, and 64 B (fp32) or 32 B (bf16) of 16-byte stores. Write-dominated,
// HBM-bound.
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
    dequant_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ sf_lin,
                   const float *__restrict__ global_scale, int64_t nblocks_total,
                   void *__restrict__ out)
{
    const float sg = *global_scale;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks_total;
         b += stride) {
        const uint2 c = __ldg(reinterpret_cast<const uint2 *>(codes) + b);
        const float fsb = e4m3_to_f32(__ldg(sf_lin + b));
        float v[16];
        const uint32_t w[2] = {c.x, c.y};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 e = e2m1x2_to_f32x2((w[i] >> (8 * j)) & 0xFFu);
                v[8 * i + 2 * j + 0] = __fmul_rn(__fmul_rn(e.x, fsb), sg);
                v[8 * i + 2 * j + 1] = __fmul_rn(__fmul_rn(e.y, fsb), sg);
            }
        if constexpr (BF16) {
            uint32_t p[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                p[j] = *reinterpret_cast<uint32_t *>(&h);
            }
            uint4 *o = reinterpret_cast<uint4 *>(out) + 2 * b;
            o[0] = make_uint4(p[0], p[1], p[2], p[3]);
            o[1] = make_uint4(p[4], p[5], p[6], p[7]);
        } else {
            float4 *o = reinterpret_cast<float4 *>(out) + 4 * b;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
}

} // namespace

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales_lin,
                              const float *global_scale, int64_t rows, int64_t cols,
                              int out_bf16, void *out, cudaStream_t s)
{
    const int64_t nblk = rows * (cols >> 4);
    if (nblk == 0)
        return cudaSuccess;
    int64_t g = (nblk + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (g > cap)
        g = cap;
    if (out_bf16)
        dequant_kernel<true><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin, global_scale,
                                                              nblk, out);
    else
        dequant_kernel<false><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin, global_scale,
                                                               nblk, out);
    return cudaGetLastError();
}

} // namespace nvfp4
