// encode_lean.cuh -- the quantizer's per-lane encode of whole 16-value blocks, written for few
// instructions a value (the encode is instruction-bound once the data is on chip): block
// maxima on packed bf16 / f16 magnitudes, the E4M3 scales of two blocks with one multiply and
// one pair conversion, codes by packed fp32 multiplies and the E2M1 pair conversion.
//
// Arithmetic (the quantizer's, unchanged): sg = amax / 2688; sb = E4M3(RN(bmax / (sg * 6)));
// code = E2M1(RN(x * RN(1 / RN(float(sb) * sg)))), with x the fp32 source value (bf16 widened
// exactly; E4M3 source times its fp32 scale, RN). The scale pair takes e4m3_of_quotient's fast
// path for both blocks at once and falls back to it per block otherwise.
#pragma once
#include <cstdint>

#include "nvfp4_encode.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {

// max(|a|, |b|) per bf16 half (the result's sign bits are not meaningful)
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// max(|a|, |b|) per f16 half (sign bits not meaningful)
__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest |x| of a 16-value bf16 block (two 16-byte vectors), as fp32 (exact).
__device__ __forceinline__ float block_absmax_bf16(const uint4 &a, const uint4 &b)
{
    uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(a.x, a.y), absmax_bf16x2(a.z, a.w)),
                               absmax_bf16x2(absmax_bf16x2(b.x, b.y), absmax_bf16x2(b.z, b.w)));
    m = absmax_bf16x2(m, __byte_perm(m, 0u, 0x1032)); // both halves: the block maximum
    return __uint_as_float((m << 16) & 0x7FFFFFFFu);
}

// Largest |x| of a 16-value fp32 block (four 16-byte vectors).
__device__ __forceinline__ float block_absmax_f32(const uint4 *v)
{
    float m[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        m[i] = fmaxf(fmaxf(fabsf(__uint_as_float(v[i].x)), fabsf(__uint_as_float(v[i].y))),
                     fmaxf(fabsf(__uint_as_float(v[i].z)), fabsf(__uint_as_float(v[i].w))));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Two E4M3 bytes (one 16-bit half of b2) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t b2)
{
    uint32_t h;
    const uint16_t in = (uint16_t)b2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
    return h;
}

// Largest |e| of a 16-value E4M3 block (one 16-byte vector) before the fp8 scale, as fp32.
__device__ __forceinline__ float block_absmax_e4m3(const uint4 &v)
{
    const uint32_t m =
        absmax_f16x2(absmax_f16x2(absmax_f16x2(e4m3x2_to_f16x2(v.x), e4m3x2_to_f16x2(v.x >> 16)),
                                  absmax_f16x2(e4m3x2_to_f16x2(v.y), e4m3x2_to_f16x2(v.y >> 16))),
                     absmax_f16x2(absmax_f16x2(e4m3x2_to_f16x2(v.z), e4m3x2_to_f16x2(v.z >> 16)),
                                  absmax_f16x2(e4m3x2_to_f16x2(v.w), e4m3x2_to_f16x2(v.w >> 16))));
    const uint32_t mm = absmax_f16x2(m, __byte_perm(m, 0u, 0x1032));
    __half_raw hr;
    hr.x = (unsigned short)(mm & 0x7FFFu);
    return __half2float(__half(hr));
}

// E4M3 scale bytes of two blocks with maxima m0, m1 (bits 0-7: m0's, bits 8-15: m1's), equal
// to e4m3_of_quotient(m0) | e4m3_of_quotient(m1) << 8. rt = RN(1 / t), t = RN(sg * 6), sg > 0.
__device__ __forceinline__ uint32_t scale_pair(float m0, float m1, float t, float rt)
{
    const float2 q = __fmul2_rn(make_float2(m0, m1), make_float2(rt, rt));
    const uint32_t u0 = __float_as_uint(q.x), u1 = __float_as_uint(q.y);
    // clear of the rounding midpoint by more than 4 ulps: |(u & 0xFFFFF) - 0x80000| > 4; in
    // range: 2^-6 <= q <= 3e38 (0x3C800000 .. 0x7F61B1E6 as bits of a non-negative float)
    const bool fast = (((u0 & 0xFFFFFu) + 0xFFF80004u) > 8u) &&
                      (((u1 & 0xFFFFFu) + 0xFFF80004u) > 8u) &&
                      (u0 - 0x3C800000u) <= 0x42E1B1E6u && (u1 - 0x3C800000u) <= 0x42E1B1E6u;
    if (fast) {
        uint16_t h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(q.y), "f"(q.x));
        return h;
    }
    return e4m3_of_quotient(m0, t, rt) | (e4m3_of_quotient(m1, t, rt) << 8);
}

// The upper bf16 of a pair as fp32, exactly (sign of zero kept), by the mixed-precision FMA
// x * 1 + (-0): the widening then runs on the FMA pipe instead of a logic operation on the
// integer pipe, which the encode keeps busy (the lower one is a shift the compiler already
// places on the FMA pipe).
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t w)
{
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;"
        : "=f"(d)
        : "h"((uint16_t)(w >> 16)), "h"((uint16_t)0x3F80), "f"(-0.0f));
    return d;
}

// E2M1 codes (low nibble first) of 8 bf16 values (one 16-byte vector) times r.
__device__ __forceinline__ uint32_t codes8_bf16(const uint4 &v, float r)
{
    const float2 rr = make_float2(r, r);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float y[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 p =
            __fmul2_rn(make_float2(__uint_as_float(w[j] << 16), bf16_hi_to_f32(w[j])), rr);
        y[2 * j] = p.x;
        y[2 * j + 1] = p.y;
    }
    return cvt_e2m1x8(y);
}

// E2M1 codes of 4 fp32 values (one 16-byte vector) times r, in the low 16 bits.
__device__ __forceinline__ uint32_t codes4_f32(const uint4 &v, float r)
{
    const float2 rr = make_float2(r, r);
    const float2 p = __fmul2_rn(make_float2(__uint_as_float(v.x), __uint_as_float(v.y)), rr);
    const float2 q = __fmul2_rn(make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), rr);
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b32 %0, {b0, b1, 0, 0};\n\t}"
        : "=r"(out)
        : "f"(p.x), "f"(p.y), "f"(q.x), "f"(q.y));
    return out;
}

// E2M1 codes of 8 E4M3 values (the bytes of w0, then of w1) times the fp8 scale s8 (RN), then
// times r (RN).
__device__ __forceinline__ uint32_t codes8_e4m3(uint32_t w0, uint32_t w1, float s8, float r)
{
    const float2 ss = make_float2(s8, s8), rr = make_float2(r, r);
    const uint32_t h[4] = {e4m3x2_to_f16x2(w0), e4m3x2_to_f16x2(w0 >> 16), e4m3x2_to_f16x2(w1),
                           e4m3x2_to_f16x2(w1 >> 16)};
    float y[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(&h[j]));
        const float2 p = __fmul2_rn(__fmul2_rn(x, ss), rr);
        y[2 * j] = p.x;
        y[2 * j + 1] = p.y;
    }
    return cvt_e2m1x8(y);
}

} // namespace nvfp4
