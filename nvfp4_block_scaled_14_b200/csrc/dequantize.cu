// dequantize.cu -- NVFP4 -> fp32 / bf16 on sm_100a.
//
// weight = E2M1 x block scale x global scale ("Qwen-Image NVFP4 on a 16 GB Ada GPU", worked
// example under the figure "First NVFP4 block, as stored in the file"), computed as
// (E2M1 * sb) * sg with two fp32 round-to-nearest multiplies; bf16 output rounds that value
// to nearest even. The page's own Ada expander does the same job with a 256-entry byte
// table in PyTorch ("Running the NVFP4 weights on Ada"); here the hardware cvt decodes two
// codes at a time.
//
// A warp takes 128 consecutive 16-value blocks per step, lane l blocks l, l + 32, l + 64,
// l + 96: every load instruction reads contiguous codes (256 B) or scales (32 B) across the
// warp and every pair of 16-byte stores writes a contiguous 1 KB (bf16) run; the four blocks'
// loads, and the next step's, are in flight together, enough bytes to cover HBM latency.
// Write-dominated, HBM-bound. With a 32-byte-aligned output each block leaves as 256-bit
// stores (one for bf16, two for fp32), so every store instruction covers whole sectors.
#include "nvfp4_internal.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void st_v8(void *p, const uint32_t (&v)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Decode one block (8 code bytes, scale sb as fp32) and store its 16 values at `o` (32-byte
// aligned when V8: 256-bit stores).
template <bool BF16, bool V8>
__device__ __forceinline__ void decode_store(uint2 c, float fsb, float sg, void *o)
{
    float v[16];
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 e = e2m1x2_to_f32x2((w[i] >> (8 * j)) & 0xFFu);
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
        if constexpr (V8) {
            st_v8(o, p);
        } else {
            uint4 *q = reinterpret_cast<uint4 *>(o);
            q[0] = make_uint4(p[0], p[1], p[2], p[3]);
            q[1] = make_uint4(p[4], p[5], p[6], p[7]);
        }
    } else if constexpr (V8) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t u[8] = {__float_as_uint(v[8 * i]), __float_as_uint(v[8 * i + 1]),
                                   __float_as_uint(v[8 * i + 2]), __float_as_uint(v[8 * i + 3]),
                                   __float_as_uint(v[8 * i + 4]), __float_as_uint(v[8 * i + 5]),
                                   __float_as_uint(v[8 * i + 6]), __float_as_uint(v[8 * i + 7])};
            st_v8(reinterpret_cast<uint8_t *>(o) + 32 * i, u);
        }
    } else {
        float4 *q = reinterpret_cast<float4 *>(o);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
}

template <bool BF16, bool V8>
__global__ void __launch_bounds__(kThreads)
    dequant_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ sf_lin,
                   const float *__restrict__ global_scale, int64_t nblocks_total,
                   void *__restrict__ out)
{
    constexpr int kOutBlk = BF16 ? 32 : 64; // output bytes per block
    const float sg = *global_scale;
    const int lane = threadIdx.x & 31;
    const int64_t nsteps = (nblocks_total + 127) >> 7; // 128-block warp steps
    const int64_t wstride = (int64_t)gridDim.x * (kThreads / 32);
    const uint2 *cb = reinterpret_cast<const uint2 *>(codes);
    uint8_t *ob = reinterpret_cast<uint8_t *>(out);
    int64_t st = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    auto load = [&](int64_t step, uint2 (&c)[4], uint32_t (&sb)[4]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t b = step * 128 + lane + 32 * j;
            if (step < nsteps && b < nblocks_total) {
                c[j] = __ldg(cb + b);
                sb[j] = __ldg(sf_lin + b);
            } else {
                c[j] = make_uint2(0u, 0u);
                sb[j] = 0u;
            }
        }
    };
    uint2 c[4], cn[4];
    uint32_t s4[4], sn[4];
    load(st, c, s4);
    for (; st < nsteps; st += wstride) {
        load(st + wstride, cn, sn); // the next step's loads in flight while this one decodes
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t b = st * 128 + lane + 32 * j;
            if (b < nblocks_total)
                decode_store<BF16, V8>(c[j], e4m3_to_f32(s4[j]), sg, ob + b * kOutBlk);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            c[j] = cn[j];
            s4[j] = sn[j];
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
    // one wave of resident CTAs (8 x 256 threads per SM), each warp 128 blocks per step
    int64_t g = (((nblk + 127) >> 7) + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap)
        g = cap;
    if (g < 1)
        g = 1;
    const bool v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    if (out_bf16 && v8)
        dequant_kernel<true, true><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin,
                                                                    global_scale, nblk, out);
    else if (out_bf16)
        dequant_kernel<true, false><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin,
                                                                     global_scale, nblk, out);
    else if (v8)
        dequant_kernel<false, true><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin,
                                                                     global_scale, nblk, out);
    else
        dequant_kernel<false, false><<<(unsigned)g, kThreads, 0, s>>>(codes, scales_lin,
                                                                      global_scale, nblk, out);
    return cudaGetLastError();
}

} // namespace nvfp4
