// internal.h -- launchers shared between the kernel files and the C ABI.
#pragma once

#include <cuda.h>  // CUtensorMap (types only; libcuda is not linked)
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace fp8moe {

// Status bits written by kernels (same values as the MOE_DEV_* macros of the
// public header).
constexpr int kDevBadExpertId = 0x1;
constexpr int kDevBadPair = 0x2;
constexpr int kDevBadOffsets = 0x4;
constexpr int kDevWaitTimeout = 0x8;

// Route kernels: tokens per ranking block (the unit of the per-block expert
// histograms the stable permutation is built from).
constexpr int kRouteTokensPerBlock = 128;

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Route workspace: status word (256 bytes), arrival counter (256 bytes),
// block histograms [ceil(T/128), E] i32, pair ranks [T*k] i32.  Returns the
// total size.
inline size_t route_ws_layout(int64_t T, int E, int k, size_t* off_arr, size_t* off_hist, size_t* off_rank)
{
    const int64_t nblocks = ceil_div64(T > 0 ? T : 1, kRouteTokensPerBlock);
    size_t o = 256;
    *off_arr = o;
    o += 256;
    *off_hist = o;
    o = align_up(o + static_cast<size_t>(nblocks) * (E > 0 ? E : 1) * 4, 256);
    *off_rank = o;
    o = align_up(o + static_cast<size_t>(T > 0 ? T : 1) * (k > 0 ? k : 1) * 4, 256);
    return o;
}

// Records a caller's timing event on s.  Inside a stream capture a plain
// record only orders the capture; the external flag makes it an event node
// that records on every replay of the graph.
inline cudaError_t record_event(void* ev, cudaStream_t s)
{
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t err = cudaStreamIsCapturing(s, &cap);
    if (err != cudaSuccess) return err;
    return cap == cudaStreamCaptureStatusActive
               ? cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), s, cudaEventRecordExternal)
               : cudaEventRecord(static_cast<cudaEvent_t>(ev), s);
}

struct DeviceInfo {
    int sm_count;
    int major, minor;
    size_t max_smem_optin;
};
// Cached per device; returns false if the current device cannot be queried.
bool device_info(DeviceInfo* out);

cudaError_t launch_quant_act(const uint16_t* x, int64_t T, int H, uint8_t* codes, float* scales, cudaStream_t s);
cudaError_t launch_encode(const float* in, int64_t n, uint8_t* out, cudaStream_t s);
// MXFP8 activations: codes [T, H] and one UE8M0 scale byte per 32 values [T, H/32].
cudaError_t launch_quant_mx(const uint16_t* x, int64_t T, int H, uint8_t* codes, uint8_t* scales, cudaStream_t s);

// Activation quantiser work carried by the route's top-k launch.
struct QuantArgs {
    const uint16_t* x;  // [T, H] BF16
    int64_t T;
    int H;
    uint8_t* codes;     // [T, H]
    float* scales;      // [T, H/128]
};

// block_hist: [ceil(T/128), E] i32; local_rank: [T*(k+shared)] i32;
// arrivals: one int (reset by the first launch, counted by the second).
// quant may be null.  shared = 1 appends the shared-expert slot (id E,
// weight 1) after the top-k: ids and w are then [T, k+1].
cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w,
                         int32_t* offsets, int32_t* sorted_pairs, int32_t* block_hist, int32_t* local_rank,
                         int* arrivals, const QuantArgs* quant, cudaStream_t s, int shared = 0);

// shared_id >= 0: slots with that id are the shared expert's rows, summed
// apart and added after the routed scaling.
cudaError_t launch_combine(const float* y, const int32_t* ids, int64_t T, int H, int k, int E, float rs,
                           float* out, uint16_t* out_bf16, int* status, cudaStream_t s, int shared_id = -1);
// Combine through a row map: out[t] = rs * sum_j y[rows[t*k + j]] over the
// slots whose row is >= 0, in slot order; rows >= y_nrows set a status bit.
cudaError_t launch_combine_rows(const float* y, int64_t y_nrows, const int32_t* rows, int64_t T, int H, int k,
                                float rs, float* out, uint16_t* out_bf16, int* status, cudaStream_t s);

// The stable permutation of pairs by key (A2 on caller-given ids): block
// ranks, expert scan, scatter (route_rank_kernel, route_scatter_kernel).
cudaError_t launch_permute(const int32_t* ids, int64_t T, int E, int k, int32_t* offsets, int32_t* sorted_pairs,
                           int32_t* block_hist, int32_t* local_rank, int* arrivals, cudaStream_t s);

struct FfnArgs {
    const uint8_t* codes;
    const float* act_scales;
    int64_t T;
    int H;
    const int32_t* topk_ids;
    const float* topk_w;
    int k;
    const int32_t* expert_offsets;
    const int32_t* sorted_pairs;
    int E;
    int I;
    const uint8_t* w_gate;
    const float* s_gate;
    const uint8_t* w_up;
    const float* s_up;
    const uint8_t* w_down;
    const float* s_down;
    float* y;
    const int32_t* y_rows;  // nullable: y row of each pair (-1: pair not written)
    int64_t y_nrows;        // rows of y when y_rows is given
    // workspace pieces
    int* status;
    uint8_t* a_sorted;   // [P, H]
    float* sa_sorted;    // [P, H/128]
    uint8_t* h_codes;    // [P, Ip]
    float* h_scales;     // [P, ceil(I/128)]
    void* const* stage_events;  // nullable: 4 cudaEvent_t for profiling
    // combine fused into the down GEMM (fuse = 1): out = rs * slot sum
    int fuse;
    float rs;
    float* out;            // [T, H]
    uint16_t* out_bf16;    // nullable
    int* cnt;              // workspace: arrival counters
    int32_t* nvalid;       // workspace: valid slots per token
    // test hook: h_codes / h_scales are caller-supplied and only the down
    // GEMM runs (no gather, no gate/up)
    int down_only;
};
size_t ffn_workspace_layout(int64_t T, int H, int I, int k, size_t* off_a, size_t* off_sa, size_t* off_h,
                            size_t* off_sh, size_t* off_cnt = nullptr, size_t* off_nv = nullptr);
// Returns cudaSuccess, or an error (including cudaErrorNotSupported when the
// tensor-map encoder cannot be obtained).
cudaError_t launch_grouped_ffn(const FfnArgs& a, cudaStream_t s);

// Row-major uint8 tensor map of `rank` (2 or 3) dims, innermost first, tile
// box 128 bytes x box_rows (x 1), 128-byte swizzle, zero fill out of bounds.
bool make_tmap_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  uint32_t box_rows);

// MXFP8 expert FFN (moe_grouped_ffn_mx): MX codes and UE8M0 scale bytes for
// activations [T, H/32], gate/up weights [E, I, H/32] and down weights
// [E, H, I/32]; the same routing inputs and y output as FfnArgs.
struct FfnMxArgs {
    const uint8_t* codes;
    const uint8_t* act_scales;  // [T, H/32]
    int64_t T;
    int H;
    const int32_t* topk_ids;
    const float* topk_w;
    int k;
    const int32_t* expert_offsets;
    const int32_t* sorted_pairs;
    int E;
    int I;
    const uint8_t* w_gate;
    const uint8_t* s_gate;  // packed [E][ceil(H/512)][I][16] (moe_mx_pack_scales)
    const uint8_t* w_up;
    const uint8_t* s_up;
    const uint8_t* w_down;
    const uint8_t* s_down;  // packed [E][ceil(I/512)][H][16]
    float* y;               // [T, k, H]
    int* status;
    uint8_t* a_sorted;      // [P, H] codes in expert order
    uint8_t* sa_sorted;     // [ceil(H/512)][P][16] scale bytes in expert order, K-group-major
    uint8_t* h_codes;       // [P, Ip]
    uint8_t* h_scales;      // [ceil(Ip/512)][P][16], the same layout
    void* const* stage_events;
    int down_only;          // 1: h_codes / h_scales are inputs; only the down GEMM runs
};
// Groups of four K blocks (512 values) of a K-wide MX operand: its scales sit
// in the workspace as [groups][rows][16 bytes].
int mx_scale_groups(int K);
// MX weight scales [E, R, K/32] -> [E][mx_scale_groups(K)][R][16] (padding
// chunks 127).
cudaError_t launch_pack_mx_scales(const uint8_t* src, int64_t E, int R, int K, uint8_t* dst, cudaStream_t s);
size_t ffn_mx_workspace_layout(int64_t T, int H, int I, int k, size_t* off_a, size_t* off_sa, size_t* off_h,
                               size_t* off_sh);
cudaError_t launch_grouped_ffn_mx(const FfnMxArgs& a, cudaStream_t s);

}  // namespace fp8moe
