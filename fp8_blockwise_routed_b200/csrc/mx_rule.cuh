// mx_rule.cuh -- the MXFP8 block rule shared by the activation quantiser and
// the MX expert FFN's requantisation epilogue (OCP Microscaling Formats:
// E4M3 elements, one UE8M0 scale per 32 values).
//   amax = max |v| over the block (NaN-propagating);
//   shared exponent se = floor(log2 amax) - 8, clamped to [-127, 127]
//   (amax = 0: se = -127); scale byte = se + 127;
//   code = E4M3_rn_satfinite(v * 2^-se);
//   a block holding NaN or Inf: scale byte 0xFF, every code 0x7F.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace fp8moe {
namespace mx {

// floor(log2 a) of a finite a > 0 (normal or subnormal), from its bits.
__device__ __forceinline__ int floor_log2_finite(float a)
{
    const uint32_t u = __float_as_uint(a);
    const int e = static_cast<int>((u >> 23) & 0xFF);
    if (e != 0) return e - 127;
    return (31 - __clz(static_cast<int>(u & 0x7FFFFF))) - 149;
}

// Shared exponent of a block with finite maximum magnitude amax.
__device__ __forceinline__ int shared_exponent(float amax)
{
    int se = amax == 0.0f ? -127 : floor_log2_finite(amax) - 8;
    return se < -127 ? -127 : (se > 127 ? 127 : se);
}

// 2^-se as a float.  For a finite FP32 maximum se <= 119, so 2^-se is a
// normal float; the subnormal branch covers se = 126, 127.
__device__ __forceinline__ float inv_scale(int se)
{
    return (-se >= -126) ? __uint_as_float(static_cast<uint32_t>(127 - se) << 23) : __uint_as_float(0x00400000u);
}

}  // namespace mx
}  // namespace fp8moe
