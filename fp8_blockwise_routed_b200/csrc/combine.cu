// combine.cu -- out[t,:] = routed_scaling * sum_j y[t,j,:] over valid slots,
// in slot order, FP32 (plus, with a shared-expert slot, that slot's row added
// after the scaling) ("Full GLM-5.3 streamed FP8 GPU prefill ...",
// "Design": routed scaling kept with the routed-expert sum; "GLM-5.3-Flash
// EXL3 on CUDA ...", commit text: routed FP32 rows).
//
// HBM-bound: each thread owns 4 consecutive columns of one token, reads the
// token's slot ids (L1-resident), streams the valid slots' float4s (up to 8
// loads in flight per thread) and writes one float4 (plus 8 bytes of BF16
// when asked).  No atomics: the sum order is
// the slot order, so a row's bits do not depend on other rows.
// Algorithmic bytes per token: (#valid slots * H + H) * 4 (+ 2H for BF16).
#include <cuda_bf16.h>

#include "internal.h"

namespace fp8moe {
namespace {

__device__ __forceinline__ float4 ld_stream_f4(const float4* p)
{
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

constexpr int kSlotBatch = 8;  // slot rows loaded together per thread

// SHARED: slots holding shared_id are the shared expert's rows, summed apart
// and added after the routed scaling (moe_combine_shared).
template <bool SHARED>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const int32_t* __restrict__ ids,
                                                      int64_t T, int H4, int k, int E, float rs,
                                                      float4* __restrict__ out, uint2* __restrict__ out_bf16,
                                                      int* __restrict__ status, int shared_id)
{
    const int64_t n = T * H4;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / H4;
        const int64_t c = i - t * H4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
        bool any_shared = false;
        // slots in batches: the batch's loads are all issued before the sums,
        // which then run in slot order over the valid slots only
        for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
            float4 v[kSlotBatch];
            bool ok[kSlotBatch], shr[kSlotBatch];
#pragma unroll
            for (int u = 0; u < kSlotBatch; ++u) {
                const int j = j0 + u;
                const int e = (j < k) ? __ldg(ids + t * k + j) : -1;
                shr[u] = SHARED && e == shared_id;
                if ((e < -1 || e >= E) && !shr[u] && c == 0) atomicOr(status, kDevBadExpertId);
                ok[u] = (e >= 0 && e < E) || shr[u];
                v[u] = ok[u] ? ld_stream_f4(y + (t * k + j) * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kSlotBatch; ++u) {
                if (!ok[u]) continue;
                if (SHARED && shr[u]) {  // the shared expert's row: summed apart, not scaled
                    any_shared = true;
                    sh.x += v[u].x;
                    sh.y += v[u].y;
                    sh.z += v[u].z;
                    sh.w += v[u].w;
                    continue;
                }
                acc.x += v[u].x;
                acc.y += v[u].y;
                acc.z += v[u].z;
                acc.w += v[u].w;
            }
        }
        float4 o = make_float4(rs * acc.x, rs * acc.y, rs * acc.z, rs * acc.w);
        if (SHARED && any_shared) o = make_float4(o.x + sh.x, o.y + sh.y, o.z + sh.z, o.w + sh.w);
        out[i] = o;
        if (out_bf16) out_bf16[i] = make_uint2(bf16x2_rn(o.x, o.y), bf16x2_rn(o.z, o.w));
    }
}

// The same sum with each slot's row taken from a row map (-1: empty slot).
__global__ void __launch_bounds__(256) combine_rows_kernel(const float4* __restrict__ y, int64_t y_nrows,
                                                           const int32_t* __restrict__ rows, int64_t T, int H4, int k,
                                                           float rs, float4* __restrict__ out,
                                                           uint2* __restrict__ out_bf16, int* __restrict__ status)
{
    const int64_t n = T * H4;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / H4;
        const int64_t c = i - t * H4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
            float4 v[kSlotBatch];
            bool ok[kSlotBatch];
#pragma unroll
            for (int u = 0; u < kSlotBatch; ++u) {
                const int j = j0 + u;
                const int64_t row = (j < k) ? __ldg(rows + t * k + j) : -1;
                if (row >= y_nrows && c == 0) atomicOr(status, kDevBadPair);
                ok[u] = row >= 0 && row < y_nrows;
                v[u] = ok[u] ? ld_stream_f4(y + row * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kSlotBatch; ++u) {
                if (!ok[u]) continue;
                acc.x += v[u].x;
                acc.y += v[u].y;
                acc.z += v[u].z;
                acc.w += v[u].w;
            }
        }
        const float4 o = make_float4(rs * acc.x, rs * acc.y, rs * acc.z, rs * acc.w);
        out[i] = o;
        if (out_bf16) out_bf16[i] = make_uint2(bf16x2_rn(o.x, o.y), bf16x2_rn(o.z, o.w));
    }
}

}  // namespace

cudaError_t launch_combine_rows(const float* y, int64_t y_nrows, const int32_t* rows, int64_t T, int H, int k,
                                float rs, float* out, uint16_t* out_bf16, int* status, cudaStream_t s)
{
    const int H4 = H / 4;
    const int64_t n = T * H4;
    if (n == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    const int64_t want = ceil_div64(n, 256);
    const int64_t cap = static_cast<int64_t>(di.sm_count) * 8 * 8;
    const int grid = static_cast<int>(want < cap ? want : cap);
    combine_rows_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(y), y_nrows, rows, T, H4, k, rs,
                                             reinterpret_cast<float4*>(out), reinterpret_cast<uint2*>(out_bf16),
                                             status);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const int32_t* ids, int64_t T, int H, int k, int E, float rs,
                           float* out, uint16_t* out_bf16, int* status, cudaStream_t s, int shared_id)
{
    const int H4 = H / 4;
    const int64_t n = T * H4;
    if (n == 0) return cudaSuccess;
    DeviceInfo di;
    if (!device_info(&di)) return cudaErrorUnknown;
    const int64_t want = ceil_div64(n, 256);
    const int64_t cap = static_cast<int64_t>(di.sm_count) * 8 * 8;
    const int grid = static_cast<int>(want < cap ? want : cap);
    if (shared_id >= 0)
        combine_kernel<true><<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(y), ids, T, H4, k, E, rs,
                                                  reinterpret_cast<float4*>(out), reinterpret_cast<uint2*>(out_bf16),
                                                  status, shared_id);
    else
        combine_kernel<false><<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(y), ids, T, H4, k, E, rs,
                                                   reinterpret_cast<float4*>(out), reinterpret_cast<uint2*>(out_bf16),
                                                   status, -1);
    return cudaGetLastError();
}

}  // namespace fp8moe
