// layer.cu -- the whole routed-expert layer behind one call, and the same
// sequence captured once into a CUDA graph ("layer plan") that is replayed
// per batch.
//
// Pages: the router chain and the layer launched as one graph ("Integration
// for GLM-4.6-FP8 and performance tune on H20", gap table row 7: the chain
// of small kernels fused and captured in-graph); one call per prompt pass
// ("GLM-5.3-Flash EXL3 on CUDA: a whole prompt pass routes its experts in
// one call").
//
// The layer is the three stream-ordered calls moe_route_quant,
// moe_grouped_ffn and moe_combine over one caller workspace, partitioned
// here.  None of them synchronises with the host or allocates, so the
// sequence can be captured as is; a plan holds the instantiated graph, and
// launching it replaces seven kernel launches, three status memsets and the
// host-side argument checks of every call by one graph launch.
#include <cstdio>
#include <new>

#include "../../include/fp8moe.h"
#include "internal.h"

namespace {

using fp8moe::align_up;

struct LayerLayout {
    size_t route, ffn, comb, codes, scales, ids, tw, offsets, sorted, y, total;
};

bool layer_layout(int64_t T, int H, int I, int E, int k, LayerLayout* L)
{
    if (T < 0 || H < 128 || H % 128 != 0 || I < 1 || E < 1 || k < 1) return false;
    const size_t t = static_cast<size_t>(T > 0 ? T : 1);
    size_t o = 0;
    auto take = [&o](size_t bytes) {
        const size_t at = o;
        o = align_up(o + (bytes > 0 ? bytes : 1), 256);
        return at;
    };
    L->route = take(moe_route_workspace_bytes(T, E, k));
    L->ffn = take(moe_ffn_workspace_bytes(T, H, I, E, k));
    L->comb = take(moe_combine_workspace_bytes());
    L->codes = take(t * H);
    L->scales = take(t * (H / 128) * 4);
    L->ids = take(t * k * 4);
    L->tw = take(t * k * 4);
    L->offsets = take(static_cast<size_t>(E + 1) * 4);
    L->sorted = take(t * k * 4);
    L->y = take(t * k * H * 4);
    L->total = o;
    return true;
}

struct LayerArgs {
    const float* logits;
    const uint16_t* x;
    int64_t T;
    int H, E, top_k, I;
    const uint8_t* w_gate;
    const float* s_gate;
    const uint8_t* w_up;
    const float* s_up;
    const uint8_t* w_down;
    const float* s_down;
    float rs;
    float* out_f32;
    uint16_t* out_bf16;
    void* ws;
    size_t ws_bytes;
};

// The three calls; stage events (nullable, 6): start, then the four marks of
// moe_grouped_ffn (gather, gate/up, down, down end), then the end.
int run_layer(const LayerArgs& a, cudaStream_t s, void* const* ev, int flags = 0)
{
    LayerLayout L;
    if (!layer_layout(a.T, a.H, a.I, a.E, a.top_k, &L)) return MOE_ERR_INVALID_ARG;
    if (!a.ws) return MOE_ERR_INVALID_ARG;
    if (a.ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(a.ws);
    auto* codes = w + L.codes;
    auto* scales = reinterpret_cast<float*>(w + L.scales);
    auto* ids = reinterpret_cast<int32_t*>(w + L.ids);
    auto* tw = reinterpret_cast<float*>(w + L.tw);
    auto* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
    auto* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
    auto* y = reinterpret_cast<float*>(w + L.y);
    if (ev && fp8moe::record_event(ev[0], s) != cudaSuccess) return MOE_ERR_CUDA;
    int r = moe_route_quant(a.logits, a.x, a.T, a.H, a.E, a.top_k, ids, tw, offsets, sorted, codes, scales,
                            w + L.route, L.ffn - L.route, s);
    if (r) return r;
    if (flags & MOE_LAYER_FUSED_COMBINE) {
        r = moe_grouped_ffn_combine(codes, scales, a.T, a.H, ids, tw, a.top_k, offsets, sorted, a.E, a.I, a.w_gate,
                                    a.s_gate, a.w_up, a.s_up, a.w_down, a.s_down, y, a.rs, a.out_f32, a.out_bf16,
                                    w + L.ffn, L.comb - L.ffn, s, ev ? ev + 1 : nullptr);
        if (r) return r;
        // no separate combine runs: its status word stays clear
        if (cudaMemsetAsync(w + L.comb, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        r = moe_grouped_ffn(codes, scales, a.T, a.H, ids, tw, a.top_k, offsets, sorted, a.E, a.I, a.w_gate,
                            a.s_gate, a.w_up, a.s_up, a.w_down, a.s_down, y, w + L.ffn, L.comb - L.ffn, s,
                            ev ? ev + 1 : nullptr);
        if (r) return r;
        r = moe_combine(y, ids, a.T, a.H, a.top_k, a.E, a.rs, a.out_f32, a.out_bf16, w + L.comb, L.codes - L.comb,
                        s);
        if (r) return r;
    }
    if (ev && fp8moe::record_event(ev[5], s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace

struct moe_layer_plan {
    cudaGraphExec_t exec;
};

extern "C" {

size_t moe_layer_workspace_bytes(int64_t T, int H, int I, int E, int top_k)
{
    LayerLayout L;
    return layer_layout(T, H, I, E, top_k, &L) ? L.total : 0;
}

int moe_layer(const float* logits, const uint16_t* x, int64_t T, int H, int E, int top_k, int I,
              const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up, const float* s_up,
              const uint8_t* w_down, const float* s_down, float routed_scaling, float* out_f32, uint16_t* out_bf16,
              void* ws, size_t ws_bytes, void* stream)
{
    const LayerArgs a{logits, x,    T,    H,     E,     top_k,          I,        w_gate, s_gate,
                      w_up,   s_up, w_down, s_down, routed_scaling, out_f32, out_bf16, ws,     ws_bytes};
    return run_layer(a, static_cast<cudaStream_t>(stream), nullptr);
}

int moe_layer_plan_create(moe_layer_plan** plan, const float* logits, const uint16_t* x, int64_t T, int H, int E,
                          int top_k, int I, const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                          const float* s_up, const uint8_t* w_down, const float* s_down, float routed_scaling,
                          float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes, void* const* stage_events)
{
    return moe_layer_plan_create_ex(plan, logits, x, T, H, E, top_k, I, w_gate, s_gate, w_up, s_up, w_down, s_down,
                                    routed_scaling, out_f32, out_bf16, ws, ws_bytes, stage_events, 0);
}

int moe_layer_plan_create_ex(moe_layer_plan** plan, const float* logits, const uint16_t* x, int64_t T, int H, int E,
                             int top_k, int I, const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                             const float* s_up, const uint8_t* w_down, const float* s_down, float routed_scaling,
                             float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes, void* const* stage_events,
                             int flags)
{
    if (flags & ~MOE_LAYER_FUSED_COMBINE) return MOE_ERR_INVALID_ARG;
    if (!plan) return MOE_ERR_INVALID_ARG;
    *plan = nullptr;
    const LayerArgs a{logits, x,    T,    H,     E,     top_k,          I,        w_gate, s_gate,
                      w_up,   s_up, w_down, s_down, routed_scaling, out_f32, out_bf16, ws,     ws_bytes};
    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
    // thread-local capture: other threads' unrelated CUDA calls stay legal
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        cudaStreamDestroy(cs);
        return MOE_ERR_CUDA;
    }
    const int r = run_layer(a, cs, stage_events, flags);
    cudaGraph_t graph = nullptr;
    const cudaError_t end = cudaStreamEndCapture(cs, &graph);
    cudaStreamDestroy(cs);
    if (r != MOE_OK || end != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return r != MOE_OK ? r : MOE_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t inst = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (inst != cudaSuccess) return MOE_ERR_CUDA;
    moe_layer_plan* p = new (std::nothrow) moe_layer_plan{exec};
    if (!p) {
        cudaGraphExecDestroy(exec);
        return MOE_ERR_CUDA;
    }
    *plan = p;
    return MOE_OK;
}

int moe_layer_plan_launch(moe_layer_plan* plan, void* stream)
{
    if (!plan) return MOE_ERR_INVALID_ARG;
    const cudaError_t err = cudaGraphLaunch(plan->exec, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

void moe_layer_plan_destroy(moe_layer_plan* plan)
{
    if (!plan) return;
    cudaGraphExecDestroy(plan->exec);
    delete plan;
}

int moe_layer_get_device_status(const void* ws, int64_t T, int H, int I, int E, int top_k, int* status_out)
{
    LayerLayout L;
    if (!ws || !status_out || !layer_layout(T, H, I, E, top_k, &L)) return MOE_ERR_INVALID_ARG;
    const uint8_t* w = static_cast<const uint8_t*>(ws);
    int acc = 0;
    for (size_t off : {L.route, L.ffn, L.comb}) {
        int v = 0;
        if (int r = moe_get_device_status(w + off, &v)) return r;
        acc |= v;
    }
    *status_out = acc;
    return MOE_OK;
}

}  // extern "C"
