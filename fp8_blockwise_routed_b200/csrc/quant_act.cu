// quant_act.cu -- BF16 -> E4M3 activation quantiser, one FP32 scale per
// 1x128 group (W8A8 activations: "Integration for GLM-4.6-FP8 and
// performance tune on H20", gap table row 6; "Full GLM-5.3 streamed FP8 GPU
// prefill ...", "Design").  The per-group rule and memory plan are in
// quant_body.cuh.  HBM-bound; algorithmic bytes per group: 256 read + 128 + 4
// written.
#include "internal.h"
#include "mx_rule.cuh"
#include "quant_body.cuh"

namespace fp8moe {
namespace {

__global__ void __launch_bounds__(256) quant_act_kernel(const uint4* __restrict__ x, int64_t n_groups,
                                                        uint8_t* __restrict__ codes, float* __restrict__ scales)
{
    quant::groups(x, n_groups, codes, scales, blockIdx.x, gridDim.x);
}

__global__ void encode_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ out)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[i] = static_cast<uint8_t>(sm100::e4m3x2(in[i], 0.0f) & 0xFFu);
}

// MXFP8 activation quantiser: one UE8M0 scale per 32 values.  Rule per
// block: amax = max|x|; shared exponent se = floor(log2(amax)) - 8, clamped
// to [-127, 127] (amax = 0: -127); scale byte se + 127; code =
// E4M3_rn_satfinite(x * 2^-se) (a product by an exact power of two; where it
// underflows the code is zero either way); a block holding NaN or Inf gets
// scale 0xFF and codes 0x7F (the rule of mx_rule.cuh).  Four lanes own a block (8 BF16 = 16 bytes each),
// a warp eight consecutive blocks per trip, kMxUnroll trips' loads in flight.
constexpr int kMxUnroll = 4;

__global__ void __launch_bounds__(256) quant_mx_kernel(const uint4* __restrict__ x, int64_t n_blocks,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales)
{
    const int lane = threadIdx.x & 31;
    const int blk = lane >> 2, sub = lane & 3;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    constexpr int kTrip = 8 * kMxUnroll;
    for (int64_t b0 = warp * kTrip; b0 < n_blocks; b0 += nwarps * kTrip) {
        uint4 raw[kMxUnroll];
#pragma unroll
        for (int u = 0; u < kMxUnroll; ++u) {
            const int64_t b = b0 + 8 * u + blk;
            raw[u] = (b < n_blocks) ? quant::ld_stream(x + b * 4 + sub) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kMxUnroll; ++u) {
            const int64_t b = b0 + 8 * u + blk;
            const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = sm100::fmax_nan(amax, fabsf(v[i]));
            amax = sm100::fmax_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            amax = sm100::fmax_nan(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
            uint2 out;
            uint8_t sc;
            if (!isfinite(amax)) {
                sc = 0xFF;
                out = make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
            } else {
                const int se = mx::shared_exponent(amax);
                sc = static_cast<uint8_t>(se + 127);
                const float f = mx::inv_scale(se);
                uint32_t p[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) p[i] = sm100::e4m3x2(v[2 * i] * f, v[2 * i + 1] * f);
                out = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
            }
            if (b < n_blocks) {
                *reinterpret_cast<uint2*>(codes + b * 32 + sub * 8) = out;
                if (sub == 0) scales[b] = sc;
            }
        }
    }
}

}  // namespace

cudaError_t launch_quant_mx(const uint16_t* x, int64_t T, int H, uint8_t* codes, uint8_t* scales, cudaStream_t s)
{
    const int64_t n_blocks = T * (H / 32);
    if (n_blocks == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    const int64_t want = ceil_div64(n_blocks, 8 * 8 * kMxUnroll);
    const int64_t cap = static_cast<int64_t>(di.sm_count) * 8 * 4;
    quant_mx_kernel<<<static_cast<int>(want < cap ? want : cap), 256, 0, s>>>(reinterpret_cast<const uint4*>(x),
                                                                               n_blocks, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_quant_act(const uint16_t* x, int64_t T, int H, uint8_t* codes, float* scales, cudaStream_t s)
{
    const int64_t n_groups = T * (H / 128);
    if (n_groups == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    const int grid = static_cast<int>(quant::blocks_for(n_groups, di.sm_count));
    quant_act_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(x), n_groups, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_encode(const float* in, int64_t n, uint8_t* out, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    const int64_t want = ceil_div64(n, 256);
    const int grid = static_cast<int>(want < 65536 ? want : 65536);
    encode_kernel<<<grid, 256, 0, s>>>(in, n, out);
    return cudaGetLastError();
}

}  // namespace fp8moe
