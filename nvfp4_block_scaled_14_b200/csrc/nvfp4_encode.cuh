// nvfp4_encode.cuh -- block-scale arithmetic shared by the quantizer and the linear layer's
// fused activation quantize, so that both produce identical codes and scales.
#pragma once
#include <cstdint>

#include "sm100_ptx.cuh"

namespace nvfp4 {

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

} // namespace nvfp4
