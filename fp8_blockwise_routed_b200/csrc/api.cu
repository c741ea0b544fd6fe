// api.cu -- the C ABI of libfp8moe.so (declared in include/fp8moe.h):
// host-side validation, workspace layout and the launch sequence.
//
// Failure policy ("Full GLM-5.3 streamed FP8 GPU prefill ...", "Design":
// explicitly reject unsupported dimensions/activation/quantisation; fail
// closed): every argument is checked before anything is enqueued, and a
// rejected call enqueues nothing.  Device-side faults are recorded in the
// status word at the start of the call's workspace, which the call clears
// (an async memset) before its first kernel.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/fp8moe.h"
#include "internal.h"

namespace fp8moe {

bool device_info(DeviceInfo* out)
{
    static DeviceInfo cache[64];
    static bool valid[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && valid[dev]) {
        *out = cache[dev];
        return true;
    }
    DeviceInfo d{};
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    d.sm_count = v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    d.major = v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    d.minor = v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    d.max_smem_optin = static_cast<size_t>(v);
    if (dev < 64) {
        cache[dev] = d;
        valid[dev] = true;
    }
    *out = d;
    return true;
}

}  // namespace fp8moe

using namespace fp8moe;

namespace {

constexpr size_t kStatusBytes = 256;

thread_local char g_last_error[256] = "";

// Record a failed CUDA call for moe_last_error() and map it to a status.
int cuda_fail(cudaError_t err, const char* where)
{
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(err),
                  static_cast<int>(err));
    return err == cudaErrorNotSupported ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common device check: an sm_100 GPU must be current.
int check_device()
{
    DeviceInfo di;
    if (!device_info(&di)) {
        std::snprintf(g_last_error, sizeof(g_last_error), "no usable CUDA device");
        return MOE_ERR_CUDA;
    }
    if (di.major != 10 || di.minor != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int clear_status(void* ws, cudaStream_t s)
{
    const cudaError_t err = cudaMemsetAsync(ws, 0, sizeof(int), s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "status clear");
}

size_t route_layout(int64_t T, int E, int k, size_t* off_arr, size_t* off_hist, size_t* off_rank)
{
    return route_ws_layout(T, E, k, off_arr, off_hist, off_rank);
}

// Shape and pointer checks shared by the MX FFN entry points.
int mx_check(int64_t T, int H, int I, int E, int top_k, const void* ws)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > MOE_MAX_EXPERTS || top_k < 1 || top_k > E || top_k > MOE_MAX_TOP_K) return MOE_ERR_INVALID_ARG;
    if (I < 128 || I > MOE_MAX_INTERMEDIATE) return MOE_ERR_INVALID_ARG;
    if (I % 32 != 0) return MOE_ERR_UNSUPPORTED;  // one scale byte per 32 intermediate columns
    if (T * top_k > (int64_t(1) << 31) - 1) return MOE_ERR_UNSUPPORTED;
    if (!ws) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_STATUS: return "MOE_ERR_DEVICE_STATUS";
    default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_abi_version(void) { return (1 << 16) | 0; }

const char* moe_last_error(void) { return g_last_error; }

size_t moe_route_workspace_bytes(int64_t T, int E, int top_k)
{
    if (T < 0 || E < 1 || top_k < 0) return 0;
    size_t a, b, c;
    return route_layout(T, E, top_k, &a, &b, &c);
}

namespace {

int route_common(const float* logits, int64_t T, int E, int top_k, int32_t* topk_ids, float* topk_w,
                 int32_t* expert_offsets, int32_t* sorted_pairs, void* ws, size_t ws_bytes, void* stream,
                 const fp8moe::QuantArgs* quant, const char* what, int shared = 0)
{
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS || top_k < 0 || top_k > E || top_k + shared > MOE_MAX_TOP_K)
        return MOE_ERR_INVALID_ARG;
    if (shared && top_k < 1) return MOE_ERR_INVALID_ARG;
    const int kp = top_k + shared;
    if (T > (int64_t(1) << 31) / (kp > 0 ? kp : 1) - 1) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets || !ws) return MOE_ERR_INVALID_ARG;
    if (T > 0 && top_k > 0 && (!logits || !topk_ids || !topk_w || !sorted_pairs)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(expert_offsets) ||
        !aligned16(sorted_pairs) || !aligned16(ws))
        return MOE_ERR_ALIGNMENT;
    size_t off_arr, off_hist, off_rank;
    if (ws_bytes < route_layout(T, E, kp, &off_arr, &off_hist, &off_rank)) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    cudaError_t err = launch_route(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs,
                                   reinterpret_cast<int32_t*>(w8 + off_hist), reinterpret_cast<int32_t*>(w8 + off_rank),
                                   reinterpret_cast<int*>(w8 + off_arr), quant, s, shared);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, what);
}

}  // namespace

int moe_route(const float* logits, int64_t T, int E, int top_k, int32_t* topk_ids, float* topk_w,
              int32_t* expert_offsets, int32_t* sorted_pairs, void* ws, size_t ws_bytes, void* stream)
{
    return route_common(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, ws_bytes, stream,
                        nullptr, "moe_route");
}

int moe_route_shared(const float* logits, int64_t T, int E, int top_k, int32_t* topk_ids, float* topk_w,
                     int32_t* expert_offsets, int32_t* sorted_pairs, void* ws, size_t ws_bytes, void* stream)
{
    return route_common(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, ws_bytes, stream,
                        nullptr, "moe_route_shared", 1);
}

int moe_route_quant(const float* logits, const uint16_t* x, int64_t T, int H, int E, int top_k, int32_t* topk_ids,
                    float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs, uint8_t* codes, float* scales,
                    void* ws, size_t ws_bytes, void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !codes || !scales)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return MOE_ERR_ALIGNMENT;
    const fp8moe::QuantArgs q{x, T, H, codes, scales};
    return route_common(logits, T, E, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, ws_bytes, stream,
                        &q, "moe_route_quant");
}

int moe_quant_act(const uint16_t* x, int64_t T, int H, uint8_t* codes, float* scales, void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !codes || !scales)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return MOE_ERR_ALIGNMENT;
    if (T == 0) return MOE_OK;
    if (int r = check_device()) return r;
    cudaError_t err = launch_quant_act(x, T, H, codes, scales, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quant_act");
}

int moe_quant_act_mx(const uint16_t* x, int64_t T, int H, uint8_t* codes, uint8_t* scales, void* stream)
{
    if (T < 0 || H < 32 || H > MOE_MAX_HIDDEN || H % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !codes || !scales)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return MOE_ERR_ALIGNMENT;
    if (T == 0) return MOE_OK;
    if (int r = check_device()) return r;
    cudaError_t err = launch_quant_mx(x, T, H, codes, scales, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quant_act_mx");
}

size_t moe_ffn_workspace_bytes(int64_t T, int H, int I, int E, int top_k)
{
    (void)E;
    if (T < 0 || H < 128 || I < 1 || top_k < 0) return 0;
    size_t a, b, c, d;
    return ffn_workspace_layout(T, H, I, top_k, &a, &b, &c, &d);
}

int moe_grouped_ffn(const uint8_t* codes, const float* act_scales, int64_t T, int H, const int32_t* topk_ids,
                    const float* topk_w, int top_k, const int32_t* expert_offsets, const int32_t* sorted_pairs,
                    int E, int I, const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                    const float* s_up, const uint8_t* w_down, const float* s_down, float* y, void* ws,
                    size_t ws_bytes, void* stream, void* const* stage_events)
{
    return moe_grouped_ffn_rows(codes, act_scales, T, H, topk_ids, topk_w, top_k, expert_offsets, sorted_pairs, E, I,
                                w_gate, s_gate, w_up, s_up, w_down, s_down, y, nullptr, 0, ws, ws_bytes, stream,
                                stage_events);
}

}  // extern "C"

namespace {

// moe_grouped_ffn and its variants: a row map for y, or the combine fused
// into the down GEMM (fuse = 1: out = routed_scaling * slot sum).
int ffn_call(const uint8_t* codes, const float* act_scales, int64_t T, int H, const int32_t* topk_ids,
             const float* topk_w, int top_k, const int32_t* expert_offsets, const int32_t* sorted_pairs, int E, int I,
             const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up, const float* s_up,
             const uint8_t* w_down, const float* s_down, float* y, const int32_t* y_rows, int64_t y_nrows, void* ws,
             size_t ws_bytes, void* stream, void* const* stage_events, int fuse, float rs, float* out,
             uint16_t* out_bf16, const char* what)
{
    if (y_rows && y_nrows < 0) return MOE_ERR_INVALID_ARG;
    if (fuse && (y_rows || (T > 0 && !out))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(out_bf16)) return MOE_ERR_ALIGNMENT;
    if (!aligned16(y_rows)) return MOE_ERR_ALIGNMENT;
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > MOE_MAX_EXPERTS || top_k < 1 || top_k > E || top_k > MOE_MAX_TOP_K) return MOE_ERR_INVALID_ARG;
    if (I < 1 || I > MOE_MAX_INTERMEDIATE) return MOE_ERR_INVALID_ARG;
    if (I % 16 != 0) return MOE_ERR_UNSUPPORTED;  // TMA row strides must be multiples of 16 bytes
    if (T * top_k > (int64_t(1) << 31) - 1) return MOE_ERR_UNSUPPORTED;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!codes || !act_scales || !topk_ids || !topk_w || !expert_offsets || !sorted_pairs || !w_gate ||
                  !s_gate || !w_up || !s_up || !w_down || !s_down || !y))
        return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs, w_gate, s_gate,
                          w_up, s_up, w_down, s_down, y, ws};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    size_t off_a, off_sa, off_h, off_sh, off_cnt, off_nv;
    if (ws_bytes < ffn_workspace_layout(T, H, I, top_k, &off_a, &off_sa, &off_h, &off_sh, &off_cnt, &off_nv))
        return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    if (T == 0) return MOE_OK;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    FfnArgs a{};
    a.codes = codes;
    a.act_scales = act_scales;
    a.T = T;
    a.H = H;
    a.topk_ids = topk_ids;
    a.topk_w = topk_w;
    a.k = top_k;
    a.expert_offsets = expert_offsets;
    a.sorted_pairs = sorted_pairs;
    a.E = E;
    a.I = I;
    a.w_gate = w_gate;
    a.s_gate = s_gate;
    a.w_up = w_up;
    a.s_up = s_up;
    a.w_down = w_down;
    a.s_down = s_down;
    a.y = y;
    a.y_rows = y_rows;
    a.y_nrows = y_nrows;
    a.status = reinterpret_cast<int*>(w8);
    a.a_sorted = w8 + off_a;
    a.sa_sorted = reinterpret_cast<float*>(w8 + off_sa);
    a.h_codes = w8 + off_h;
    a.h_scales = reinterpret_cast<float*>(w8 + off_sh);
    a.stage_events = stage_events;
    a.fuse = fuse;
    a.rs = rs;
    a.out = out;
    a.out_bf16 = out_bf16;
    a.cnt = reinterpret_cast<int*>(w8 + off_cnt);
    a.nvalid = reinterpret_cast<int32_t*>(w8 + off_nv);
    cudaError_t err = launch_grouped_ffn(a, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, what);
}

}  // namespace

extern "C" {

int moe_grouped_ffn_rows(const uint8_t* codes, const float* act_scales, int64_t T, int H, const int32_t* topk_ids,
                         const float* topk_w, int top_k, const int32_t* expert_offsets, const int32_t* sorted_pairs,
                         int E, int I, const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                         const float* s_up, const uint8_t* w_down, const float* s_down, float* y,
                         const int32_t* y_rows, int64_t y_nrows, void* ws, size_t ws_bytes, void* stream,
                         void* const* stage_events)
{
    return ffn_call(codes, act_scales, T, H, topk_ids, topk_w, top_k, expert_offsets, sorted_pairs, E, I, w_gate,
                    s_gate, w_up, s_up, w_down, s_down, y, y_rows, y_nrows, ws, ws_bytes, stream, stage_events, 0,
                    0.f, nullptr, nullptr, "moe_grouped_ffn");
}

int moe_grouped_ffn_combine(const uint8_t* codes, const float* act_scales, int64_t T, int H,
                            const int32_t* topk_ids, const float* topk_w, int top_k, const int32_t* expert_offsets,
                            const int32_t* sorted_pairs, int E, int I, const uint8_t* w_gate, const float* s_gate,
                            const uint8_t* w_up, const float* s_up, const uint8_t* w_down, const float* s_down,
                            float* y, float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws,
                            size_t ws_bytes, void* stream, void* const* stage_events)
{
    return ffn_call(codes, act_scales, T, H, topk_ids, topk_w, top_k, expert_offsets, sorted_pairs, E, I, w_gate,
                    s_gate, w_up, s_up, w_down, s_down, y, nullptr, 0, ws, ws_bytes, stream, stage_events, 1,
                    routed_scaling, out_f32, out_bf16, "moe_grouped_ffn_combine");
}

size_t moe_combine_workspace_bytes(void) { return kStatusBytes; }

int moe_combine(const float* y, const int32_t* topk_ids, int64_t T, int H, int top_k, int E, float routed_scaling,
                float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes, void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (top_k < 0 || top_k > MOE_MAX_TOP_K || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (!ws || (T > 0 && !out_f32) || (T > 0 && top_k > 0 && (!y || !topk_ids))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(topk_ids) || !aligned16(out_f32) || !aligned16(out_bf16) || !aligned16(ws))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    cudaError_t err = launch_combine(y, topk_ids, T, H, top_k, E, routed_scaling, out_f32, out_bf16,
                                     static_cast<int*>(ws), s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine");
}

int moe_combine_shared(const float* y, const int32_t* topk_ids, int64_t T, int H, int top_k, int E,
                       float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                       void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > MOE_MAX_TOP_K || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (!ws || (T > 0 && (!out_f32 || !y || !topk_ids))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(topk_ids) || !aligned16(out_f32) || !aligned16(out_bf16) || !aligned16(ws))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    cudaError_t err = launch_combine(y, topk_ids, T, H, top_k, E, routed_scaling, out_f32, out_bf16,
                                     static_cast<int*>(ws), s, E);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine_shared");
}

int moe_combine_rows(const float* y, int64_t y_nrows, const int32_t* rows, int64_t T, int H, int top_k,
                     float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes, void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (top_k < 0 || top_k > MOE_MAX_TOP_K || y_nrows < 0) return MOE_ERR_INVALID_ARG;
    if (!ws || (T > 0 && !out_f32) || (T > 0 && top_k > 0 && (!rows || (y_nrows > 0 && !y))))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(rows) || !aligned16(out_f32) || !aligned16(out_bf16) || !aligned16(ws))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    cudaError_t err = launch_combine_rows(y, y_nrows, rows, T, H, top_k, routed_scaling, out_f32, out_bf16,
                                          static_cast<int*>(ws), s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine_rows");
}

int moe_get_device_status(const void* ws, int* status_out)
{
    if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
    cudaError_t err = cudaDeviceSynchronize();
    if (err != cudaSuccess) return cuda_fail(err, "moe_get_device_status sync");
    int v = 0;
    err = cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost);
    if (err != cudaSuccess) return cuda_fail(err, "moe_get_device_status copy");
    *status_out = v;
    return MOE_OK;
}

int moe_debug_encode(const float* in, int64_t n, uint8_t* out, void* stream)
{
    if (n < 0 || (n > 0 && (!in || !out))) return MOE_ERR_INVALID_ARG;
    if (int r = check_device()) return r;
    cudaError_t err = launch_encode(in, n, out, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_debug_encode");
}

int moe_debug_grouped_down(const uint8_t* h_codes, const float* h_scales, int64_t T, int H, int top_k,
                           const float* topk_w, const int32_t* expert_offsets, const int32_t* sorted_pairs, int E,
                           int I, const uint8_t* w_down, const float* s_down, float* y, void* ws, size_t ws_bytes,
                           void* stream)
{
    if (T < 0 || H < 128 || H > MOE_MAX_HIDDEN || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > MOE_MAX_EXPERTS || top_k < 1 || top_k > E || top_k > MOE_MAX_TOP_K) return MOE_ERR_INVALID_ARG;
    if (I < 1 || I > MOE_MAX_INTERMEDIATE) return MOE_ERR_INVALID_ARG;
    if (I % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T * top_k > (int64_t(1) << 31) - 1) return MOE_ERR_UNSUPPORTED;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!h_codes || !h_scales || !topk_w || !expert_offsets || !sorted_pairs || !w_down || !s_down || !y))
        return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {h_codes, h_scales, topk_w, expert_offsets, sorted_pairs, w_down, s_down, y, ws};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    if (T == 0) return MOE_OK;
    FfnArgs a{};
    a.T = T;
    a.H = H;
    a.topk_w = topk_w;
    a.k = top_k;
    a.expert_offsets = expert_offsets;
    a.sorted_pairs = sorted_pairs;
    a.E = E;
    a.I = I;
    a.w_down = w_down;
    a.s_down = s_down;
    a.y = y;
    a.status = static_cast<int*>(ws);
    a.h_codes = const_cast<uint8_t*>(h_codes);
    a.h_scales = const_cast<float*>(h_scales);
    a.down_only = 1;
    cudaError_t err = launch_grouped_ffn(a, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_debug_grouped_down");
}


size_t moe_mx_packed_scales_bytes(int64_t E, int R, int K)
{
    if (E < 0 || R < 1 || K < 32 || K % 32 != 0) return 0;
    return static_cast<size_t>(E) * mx_scale_groups(K) * R * 16;
}

int moe_mx_pack_scales(const uint8_t* src, int64_t E, int R, int K, uint8_t* dst, void* stream)
{
    if (E < 0 || R < 1 || K < 32 || K % 32 != 0) return MOE_ERR_INVALID_ARG;
    if (E > 0 && (!src || !dst)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(dst)) return MOE_ERR_ALIGNMENT;
    if (E == 0) return MOE_OK;
    if (int r = check_device()) return r;
    cudaError_t err = launch_pack_mx_scales(src, E, R, K, dst, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_mx_pack_scales");
}

size_t moe_ffn_mx_workspace_bytes(int64_t T, int H, int I, int E, int top_k)
{
    (void)E;
    if (T < 0 || H < 128 || I < 1 || top_k < 0) return 0;
    size_t a, b, c, d;
    return ffn_mx_workspace_layout(T, H, I, top_k, &a, &b, &c, &d);
}

int moe_grouped_ffn_mx(const uint8_t* codes, const uint8_t* act_scales, int64_t T, int H, const int32_t* topk_ids,
                       const float* topk_w, int top_k, const int32_t* expert_offsets, const int32_t* sorted_pairs,
                       int E, int I, const uint8_t* w_gate, const uint8_t* s_gate, const uint8_t* w_up,
                       const uint8_t* s_up, const uint8_t* w_down, const uint8_t* s_down, float* y, void* ws,
                       size_t ws_bytes, void* stream, void* const* stage_events)
{
    if (int r = mx_check(T, H, I, E, top_k, ws)) return r;
    if (T > 0 && (!codes || !act_scales || !topk_ids || !topk_w || !expert_offsets || !sorted_pairs || !w_gate ||
                  !s_gate || !w_up || !s_up || !w_down || !s_down || !y))
        return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs, w_gate, s_gate,
                          w_up, s_up, w_down, s_down, y, ws};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    size_t off_a, off_sa, off_h, off_sh;
    if (ws_bytes < ffn_mx_workspace_layout(T, H, I, top_k, &off_a, &off_sa, &off_h, &off_sh))
        return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    if (T == 0) return MOE_OK;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    FfnMxArgs a{};
    a.codes = codes;
    a.act_scales = act_scales;
    a.T = T;
    a.H = H;
    a.topk_ids = topk_ids;
    a.topk_w = topk_w;
    a.k = top_k;
    a.expert_offsets = expert_offsets;
    a.sorted_pairs = sorted_pairs;
    a.E = E;
    a.I = I;
    a.w_gate = w_gate;
    a.s_gate = s_gate;
    a.w_up = w_up;
    a.s_up = s_up;
    a.w_down = w_down;
    a.s_down = s_down;
    a.y = y;
    a.status = reinterpret_cast<int*>(w8);
    a.a_sorted = w8 + off_a;
    a.sa_sorted = w8 + off_sa;
    a.h_codes = w8 + off_h;
    a.h_scales = w8 + off_sh;
    a.stage_events = stage_events;
    cudaError_t err = launch_grouped_ffn_mx(a, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_ffn_mx");
}

int moe_ffn_mx_intermediate(const void* ws, int64_t T, int H, int I, int top_k, const uint8_t** h_codes,
                            const uint8_t** h_scales)
{
    if (!ws || !h_codes || !h_scales || T < 0 || H < 128 || I < 1 || top_k < 1) return MOE_ERR_INVALID_ARG;
    size_t off_a, off_sa, off_h, off_sh;
    ffn_mx_workspace_layout(T, H, I, top_k, &off_a, &off_sa, &off_h, &off_sh);
    *h_codes = static_cast<const uint8_t*>(ws) + off_h;
    *h_scales = static_cast<const uint8_t*>(ws) + off_sh;
    return MOE_OK;
}

int moe_debug_grouped_down_mx(const uint8_t* h_codes, const uint8_t* h_scales, int64_t T, int H, int top_k,
                              const float* topk_w, const int32_t* expert_offsets, const int32_t* sorted_pairs, int E,
                              int I, const uint8_t* w_down, const uint8_t* s_down, float* y, void* ws,
                              size_t ws_bytes, void* stream)
{
    if (int r = mx_check(T, H, I, E, top_k, ws)) return r;
    if (T > 0 && (!h_codes || !h_scales || !topk_w || !expert_offsets || !sorted_pairs || !w_down || !s_down || !y))
        return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {h_codes, h_scales, topk_w, expert_offsets, sorted_pairs, w_down, s_down, y, ws};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (int r = check_device()) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int r = clear_status(ws, s)) return r;
    if (T == 0) return MOE_OK;
    FfnMxArgs a{};
    a.T = T;
    a.H = H;
    a.topk_w = topk_w;
    a.k = top_k;
    a.expert_offsets = expert_offsets;
    a.sorted_pairs = sorted_pairs;
    a.E = E;
    a.I = I;
    a.w_down = w_down;
    a.s_down = s_down;
    a.y = y;
    a.status = static_cast<int*>(ws);
    a.h_codes = const_cast<uint8_t*>(h_codes);
    a.h_scales = const_cast<uint8_t*>(h_scales);
    a.down_only = 1;
    cudaError_t err = launch_grouped_ffn_mx(a, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_debug_grouped_down_mx");
}

int moe_ffn_intermediate(const void* ws, int64_t T, int H, int I, int top_k, const uint8_t** h_codes,
                         const float** h_scales)
{
    if (!ws || !h_codes || !h_scales || T < 0 || H < 128 || I < 1 || top_k < 1) return MOE_ERR_INVALID_ARG;
    size_t off_a, off_sa, off_h, off_sh;
    ffn_workspace_layout(T, H, I, top_k, &off_a, &off_sa, &off_h, &off_sh);
    *h_codes = static_cast<const uint8_t*>(ws) + off_h;
    *h_scales = reinterpret_cast<const float*>(static_cast<const uint8_t*>(ws) + off_sh);
    return MOE_OK;
}

}  // extern "C"
