// quant_act.cu -- BF16 -> E4M3 activation quantiser, one FP32 scale per
// 1x128 group (W8A8 activations: "Integration for GLM-4.6-FP8 and
// performance tune on H20", gap table row 6; "Full GLM-5.3 streamed FP8 GPU
// prefill ...", "Design").  The per-group rule and memory plan are in
// quant_body.cuh.  HBM-bound; algorithmic bytes per group: 256 read + 128 + 4
// written.
#include "internal.h"
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

}  // namespace

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
