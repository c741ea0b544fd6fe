// quant_body.cuh -- the activation quantiser's per-group body, shared by
// quant_act_kernel and the fused route+quantise launch.
//
// Rule per 1x128 group: amax = max|x|; s = amax/448 (the IEEE quotient);
// s == 0 -> 1; code = E4M3_rn_satfinite(x/s) (the IEEE quotient); a group
// holding NaN/Inf gets s = NaN and codes 0x7F.  Both quotients are formed
// below without a divide, by corrected reciprocal products that give the
// same scales and codes.  No flush-to-zero (built without fast-math).
//
// A quarter warp owns one group: each lane loads two 16-byte vectors (16
// BF16), the 8 lanes reduce amax with shuffles, each lane stores 16 code
// bytes, lane 0 of the quarter stores the scale.  Loads are fully coalesced
// (a warp reads 1 KB of contiguous groups), stores 512 contiguous bytes.
#pragma once

#include "sm100.cuh"

namespace fp8moe {
namespace quant {

__device__ __forceinline__ uint4 ld_stream(const uint4* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kUnroll = 4;  // groups per half-warp per trip, loads issued together

// x / s without the divide: with y = RN(1/s) and q = RN(x*y), the remainder
// r = s*q - x is exact in one FMA and RN(q - r*y) is the correctly rounded
// quotient (Markstein's correction step, P. Markstein, IBM J. Res. Dev.
// 34(1), 1990), as long as r does not underflow.  For BF16 x and
// s = RN(amax/448) with |x| <= amax, an exhaustive comparison with the IEEE
// divide over every such pair with s >= 2^-100 finds equal E4M3 codes
// everywhere: the two floats differ only where both are below 2^-11 in
// magnitude, i.e. both encode to zero.  The sign is copied from x so that
// zero quotients keep it (-0/s = -0).  Smaller scales keep the divide.
constexpr float kExactQuotientMinScale = 0x1p-100f;

__device__ __forceinline__ float quotient(float x, float s, float y)
{
    const float q = __fmul_rn(x, y);
    const float r = __fmaf_rn(s, q, -x);
    return copysignf(__fmaf_rn(-r, y, q), x);
}

// s = RN(amax / 448) by the same correction with y = RN(1/448): for every
// finite non-negative BF16 amax (the group maximum is one of the group's
// BF16 values) it equals the IEEE quotient, subnormal results included
// (exhaustive host comparison over all 32,640 values).
constexpr float kInv448 = 0x1.24924ap-9f;

__device__ __forceinline__ float group_scale(float amax)
{
    const float q = __fmul_rn(amax, kInv448);
    const float r = __fmaf_rn(448.0f, q, -amax);
    return __fmaf_rn(-r, kInv448, q);
}

// The same quotient for two values at once on packed FP32 pairs
// (mul.rn.f32x2 / fma.rn.f32x2 round each element exactly as the scalar
// operations do).  With rn = RN(-s*q + x) = -r (r is exact, and RN is
// symmetric), d = RN(rn*y + q) is the value above; only the sign of a zero
// d can differ, and the copy of x's sign fixes that.
__device__ __forceinline__ void quotient2(float x0, float x1, float s, float y, float& d0, float& d1)
{
    asm("{\n\t.reg .b64 X, NS, Y, Q, RN, D;\n\t"
        "mov.b64 X, {%2, %3};\n\t"
        "mov.b64 NS, {%4, %4};\n\t"
        "mov.b64 Y, {%5, %5};\n\t"
        "mul.rn.f32x2 Q, X, Y;\n\t"
        "fma.rn.f32x2 RN, NS, Q, X;\n\t"
        "fma.rn.f32x2 D, RN, Y, Q;\n\t"
        "mov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(x0), "f"(x1), "f"(-s), "f"(y));
    d0 = copysignf(d0, x0);
    d1 = copysignf(d1, x1);
}

constexpr int kLanesPerGroup = 8;  // a quarter warp owns a group: 16 values per lane
constexpr int kGroupsPerWarp = 32 / kLanesPerGroup;

// Quantises groups [0, n_groups) with the warps of `nblocks` blocks of
// blockDim.x threads, this thread belonging to block `block`.  A quarter
// warp owns a group (each lane 16 values: two 16-byte loads, one 16-byte
// code store), so the per-group work that every lane repeats (the scale and
// its reciprocal) is paid by 8 lanes, and the amax reduction takes three
// shuffle rounds.  Per trip a warp covers kGroupsPerWarp*kUnroll consecutive
// groups; its loads are issued before any of them is reduced.
__device__ __forceinline__ void groups(const uint4* __restrict__ x, int64_t n_groups, uint8_t* __restrict__ codes,
                                       float* __restrict__ scales, int64_t block, int64_t nblocks)
{
    const int lane = threadIdx.x & 31;
    const int quarter = lane / kLanesPerGroup;
    const int sub = lane % kLanesPerGroup;
    const int64_t warp = (block * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (nblocks * blockDim.x) >> 5;
    constexpr int kTrip = kGroupsPerWarp * kUnroll;

    for (int64_t g0 = warp * kTrip; g0 < n_groups; g0 += nwarps * kTrip) {
        uint4 raw[kUnroll][2];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + kGroupsPerWarp * u + quarter;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                raw[u][h] = (g < n_groups) ? ld_stream(x + g * 16 + sub * 2 + h) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = g0 + kGroupsPerWarp * u + quarter;
            const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                   raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
            float v[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            // NaN-propagating max: a NaN or Inf anywhere in the group leaves
            // amax non-finite, so one test after the reduction finds it
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = sm100::fmax_nan(amax, fabsf(v[i]));
#pragma unroll
            for (int off = kLanesPerGroup / 2; off > 0; off >>= 1)
                amax = sm100::fmax_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
            const bool bad = !isfinite(amax);
            float s = group_scale(amax);
            if (s == 0.0f) s = 1.0f;
            uint4 out;
            if (bad) {
                s = __int_as_float(0x7FC00000);
                out = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            } else if (s >= kExactQuotientMinScale) {
                const float y = __frcp_rn(s);
                float d[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) quotient2(v[2 * i], v[2 * i + 1], s, y, d[2 * i], d[2 * i + 1]);
                uint32_t p[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) p[i] = sm100::e4m3x2(d[2 * i], d[2 * i + 1]);
                out = make_uint4(p[0] | (p[1] << 16), p[2] | (p[3] << 16), p[4] | (p[5] << 16), p[6] | (p[7] << 16));
            } else {  // groups whose amax is below 448 * 2^-100
                uint32_t p[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    p[i] = sm100::e4m3x2(__fdiv_rn(v[2 * i], s), __fdiv_rn(v[2 * i + 1], s));
                out = make_uint4(p[0] | (p[1] << 16), p[2] | (p[3] << 16), p[4] | (p[5] << 16), p[6] | (p[7] << 16));
            }
            if (g < n_groups) {
                *reinterpret_cast<uint4*>(codes + g * 128 + sub * 16) = out;
                if (sub == 0) scales[g] = s;
            }
        }
    }
}

// Blocks of 256 threads that quantise n_groups: one trip of every warp over
// the groups when the grid allows it, at most a few waves of 8 resident
// blocks per SM (grid-stride beyond that).
inline int64_t blocks_for(int64_t n_groups, int sm_count)
{
    const int64_t want = (n_groups + 8 * kGroupsPerWarp * kUnroll - 1) / (8 * kGroupsPerWarp * kUnroll);
    const int64_t cap = static_cast<int64_t>(sm_count) * 8 * 4;
    return want < cap ? want : cap;
}

}  // namespace quant
}  // namespace fp8moe
