"""Python binding of libfp8moe.so: the B200 routed-MoE FP8 blockwise (W8A8)
prefill path.

Functions named after the C ABI (include/fp8moe.h) marshal torch tensors
into pointers and the current CUDA stream; every step of the path runs in the
library's CUDA kernels.  PyTorch provides device memory and streams only.
There is no fallback: if the library is missing or the device is not an
sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8moe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "fp8moe.h")

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_ALIGNMENT",
          4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_DEVICE_STATUS"}
DEV_BAD_EXPERT_ID, DEV_BAD_PAIR, DEV_BAD_OFFSETS, DEV_WAIT_TIMEOUT = 0x1, 0x2, 0x4, 0x8

_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        super().__init__(f"{what} failed: {STATUS.get(code, code)}" + (f" ({detail})" if detail else ""))
        self.code = code


def declared_functions() -> list[str]:
    """Names of the functions the public header declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m fp8_blockwise_routed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [i32]
        L.moe_abi_version.restype = i32
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        L.moe_route_workspace_bytes.restype = sz
        L.moe_route_workspace_bytes.argtypes = [i64, i32, i32]
        L.moe_route.restype = i32
        L.moe_route.argtypes = [P, i64, i32, i32, P, P, P, P, P, sz, P]
        L.moe_route_noalloc.restype = i32
        L.moe_route_noalloc.argtypes = [P, i64, i32, i32, P, P, P, P, P]
        L.moe_route_noalloc_error.restype = ctypes.c_char_p
        L.moe_route_noalloc_error.argtypes = []
        L.moe_quant_act_mx.restype = i32
        L.moe_quant_act_mx.argtypes = [P, i64, i32, P, P, P]
        L.moe_quant_act.restype = i32
        L.moe_quant_act.argtypes = [P, i64, i32, P, P, P]
        L.moe_layer_workspace_bytes.restype = sz
        L.moe_layer_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
        L.moe_layer.restype = i32
        L.moe_layer.argtypes = [P, P, i64, i32, i32, i32, i32, P, P, P, P, P, P, ctypes.c_float, P, P, P, sz, P]
        L.moe_layer_plan_create.restype = i32
        L.moe_layer_plan_create.argtypes = [ctypes.POINTER(ctypes.c_void_p), P, P, i64, i32, i32, i32, i32,
                                            P, P, P, P, P, P, ctypes.c_float, P, P, P, sz, P]
        L.moe_layer_plan_launch.restype = i32
        L.moe_layer_plan_launch.argtypes = [P, P]
        L.moe_layer_plan_destroy.restype = None
        L.moe_layer_plan_destroy.argtypes = [P]
        L.moe_layer_get_device_status.restype = i32
        L.moe_layer_get_device_status.argtypes = [P, i64, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int)]
        L.moe_ep_plan_workspace_bytes.restype = sz
        L.moe_ep_plan_workspace_bytes.argtypes = [i64, i32, i32]
        L.moe_ep_plan.restype = i32
        L.moe_ep_plan.argtypes = [P, i64, i32, i32, i32, i32, i64, P, P, P, P, P, P, sz, P]
        L.moe_permute.restype = i32
        L.moe_permute.argtypes = [P, i64, i32, i32, P, P, P, sz, P]
        L.moe_grouped_ffn_rows.restype = i32
        L.moe_grouped_ffn_rows.argtypes = [P, P, i64, i32, P, P, i32, P, P, i32, i32, P, P, P, P, P, P, P, P, i64,
                                           P, sz, P, P]
        L.moe_combine_rows.restype = i32
        L.moe_combine_rows.argtypes = [P, i64, P, i64, i32, i32, ctypes.c_float, P, P, P, sz, P]
        L.moe_grouped_ffn_combine.restype = i32
        L.moe_grouped_ffn_combine.argtypes = [P, P, i64, i32, P, P, i32, P, P, i32, i32, P, P, P, P, P, P, P,
                                              ctypes.c_float, P, P, P, sz, P, P]
        L.moe_layer_plan_create_ex.restype = i32
        L.moe_layer_plan_create_ex.argtypes = [ctypes.POINTER(ctypes.c_void_p), P, P, i64, i32, i32, i32, i32,
                                               P, P, P, P, P, P, ctypes.c_float, P, P, P, sz, P, i32]
        L.moe_route_shared.restype = i32
        L.moe_route_shared.argtypes = [P, i64, i32, i32, P, P, P, P, P, sz, P]
        L.moe_combine_shared.restype = i32
        L.moe_combine_shared.argtypes = [P, P, i64, i32, i32, i32, ctypes.c_float, P, P, P, sz, P]
        L.moe_route_quant.restype = i32
        L.moe_route_quant.argtypes = [P, P, i64, i32, i32, i32, P, P, P, P, P, P, P, sz, P]
        L.moe_ffn_workspace_bytes.restype = sz
        L.moe_ffn_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
        L.moe_grouped_ffn.restype = i32
        L.moe_grouped_ffn.argtypes = [P, P, i64, i32, P, P, i32, P, P, i32, i32,
                                      P, P, P, P, P, P, P, P, sz, P, P]
        L.moe_combine_workspace_bytes.restype = sz
        L.moe_combine_workspace_bytes.argtypes = []
        L.moe_combine.restype = i32
        L.moe_combine.argtypes = [P, P, i64, i32, i32, i32, ctypes.c_float, P, P, P, sz, P]
        L.moe_get_device_status.restype = i32
        L.moe_get_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
        L.moe_debug_encode.restype = i32
        L.moe_debug_encode.argtypes = [P, i64, P, P]
        L.moe_debug_grouped_down.restype = i32
        L.moe_debug_grouped_down.argtypes = [P, P, i64, i32, i32, P, P, P, i32, i32, P, P, P, P, sz, P]
        L.moe_ffn_intermediate.restype = i32
        L.moe_ffn_intermediate.argtypes = [P, i64, i32, i32, i32, ctypes.POINTER(ctypes.c_void_p),
                                           ctypes.POINTER(ctypes.c_void_p)]
        L.moe_mx_packed_scales_bytes.restype = sz
        L.moe_mx_packed_scales_bytes.argtypes = [i64, i32, i32]
        L.moe_mx_pack_scales.restype = i32
        L.moe_mx_pack_scales.argtypes = [P, i64, i32, i32, P, P]
        L.moe_ffn_mx_workspace_bytes.restype = sz
        L.moe_ffn_mx_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
        L.moe_grouped_ffn_mx.restype = i32
        L.moe_grouped_ffn_mx.argtypes = [P, P, i64, i32, P, P, i32, P, P, i32, i32,
                                         P, P, P, P, P, P, P, P, sz, P, P]
        L.moe_ffn_mx_intermediate.restype = i32
        L.moe_ffn_mx_intermediate.argtypes = [P, i64, i32, i32, i32, ctypes.POINTER(ctypes.c_void_p),
                                              ctypes.POINTER(ctypes.c_void_p)]
        L.moe_debug_grouped_down_mx.restype = i32
        L.moe_debug_grouped_down_mx.argtypes = [P, P, i64, i32, i32, P, P, P, i32, i32, P, P, P, P, sz, P]
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code: int, what: str):
    if code != 0:
        detail = lib().moe_last_error().decode() if code in (2, 5) else ""
        raise MoeError(code, what, detail)


# ------------------------------------------------------------------ sizes

def moe_route_workspace_bytes(T: int, E: int, top_k: int) -> int:
    return int(lib().moe_route_workspace_bytes(T, E, top_k))


def moe_ffn_workspace_bytes(T: int, H: int, I: int, E: int, top_k: int) -> int:
    return int(lib().moe_ffn_workspace_bytes(T, H, I, E, top_k))


def moe_combine_workspace_bytes() -> int:
    return int(lib().moe_combine_workspace_bytes())


# ------------------------------------------------------------------ calls

def moe_route(logits, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, stream=None):
    T, E = logits.shape
    _check(lib().moe_route(_p(logits), T, E, top_k, _p(topk_ids), _p(topk_w), _p(expert_offsets),
                           _p(sorted_pairs), _p(ws), ws.numel() * ws.element_size(), _s(stream)), "moe_route")


def moe_route_noalloc(logits, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, stream=None):
    """moe_route for callers that cannot allocate device memory: no workspace;
    the library's static device scratch is used instead (calls that overlap
    on the GPU race; see the header)."""
    T, E = logits.shape
    code = lib().moe_route_noalloc(_p(logits), T, E, top_k, _p(topk_ids), _p(topk_w), _p(expert_offsets),
                                   _p(sorted_pairs), _s(stream))
    if code != 0:
        raise MoeError(code, "moe_route_noalloc", lib().moe_route_noalloc_error().decode())


def moe_quant_act(x, codes, scales, stream=None):
    T, H = x.shape
    _check(lib().moe_quant_act(_p(x), T, H, _p(codes), _p(scales), _s(stream)), "moe_quant_act")


def moe_quant_act_mx(x, codes, scales, stream=None):
    """BF16 [T,H] -> MXFP8 codes uint8 [T,H] and UE8M0 scale bytes [T,H/32]."""
    T, H = x.shape
    _check(lib().moe_quant_act_mx(_p(x), T, H, _p(codes), _p(scales), _s(stream)), "moe_quant_act_mx")


def moe_route_quant(logits, x, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, codes, scales, ws,
                    stream=None):
    """moe_route and moe_quant_act in one call (the quantiser rides in the
    router's first launch); same results as the two calls."""
    T, E = logits.shape
    H = x.shape[1]
    assert x.shape[0] == T
    _check(lib().moe_route_quant(_p(logits), _p(x), T, H, E, top_k, _p(topk_ids), _p(topk_w), _p(expert_offsets),
                                 _p(sorted_pairs), _p(codes), _p(scales), _p(ws), ws.numel() * ws.element_size(),
                                 _s(stream)), "moe_route_quant")


def moe_grouped_ffn(codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs,
                    w_gate, s_gate, w_up, s_up, w_down, s_down, y, ws, stream=None, stage_events=None):
    """stage_events: None or 4 torch.cuda.Event objects (already recorded
    once, so that their handles exist) marking gather / gate-up / down / end."""
    T, H = codes.shape
    E, I, _ = w_gate.shape
    top_k = topk_ids.shape[1]
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * 4)(*[e.cuda_event for e in stage_events])
    _check(lib().moe_grouped_ffn(_p(codes), _p(act_scales), T, H, _p(topk_ids), _p(topk_w), top_k,
                                 _p(expert_offsets), _p(sorted_pairs), E, I, _p(w_gate), _p(s_gate),
                                 _p(w_up), _p(s_up), _p(w_down), _p(s_down), _p(y), _p(ws),
                                 ws.numel() * ws.element_size(), _s(stream), ev), "moe_grouped_ffn")


def moe_mx_pack_scales(src, stream=None):
    """MX weight scales [E, R, K/32] uint8 (CUDA) -> the packed layout the MX
    FFN reads: a new uint8 tensor [E, ceil(K/512), R, 16]."""
    E, R, C = src.shape
    K = C * 32
    G = (K + 511) // 512
    assert int(lib().moe_mx_packed_scales_bytes(E, R, K)) == E * G * R * 16
    dst = torch.empty((E, G, R, 16), dtype=torch.uint8, device=src.device)
    _check(lib().moe_mx_pack_scales(_p(src.contiguous()), E, R, K, _p(dst), _s(stream)), "moe_mx_pack_scales")
    return dst


def moe_ffn_mx_workspace_bytes(T: int, H: int, I: int, E: int, top_k: int) -> int:
    return int(lib().moe_ffn_mx_workspace_bytes(T, H, I, E, top_k))


def moe_grouped_ffn_mx(codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs,
                       w_gate, s_gate, w_up, s_up, w_down, s_down, y, ws, stream=None, stage_events=None):
    """The MXFP8 experts: uint8 codes with uint8 UE8M0 scale bytes per 32
    values (act_scales [T, H/32]; s_gate, s_up, s_down as moe_mx_pack_scales
    returns them)."""
    T, H = codes.shape
    E, I, _ = w_gate.shape
    top_k = topk_ids.shape[1]
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * 4)(*[e.cuda_event for e in stage_events])
    _check(lib().moe_grouped_ffn_mx(_p(codes), _p(act_scales), T, H, _p(topk_ids), _p(topk_w), top_k,
                                    _p(expert_offsets), _p(sorted_pairs), E, I, _p(w_gate), _p(s_gate),
                                    _p(w_up), _p(s_up), _p(w_down), _p(s_down), _p(y), _p(ws),
                                    ws.numel() * ws.element_size(), _s(stream), ev), "moe_grouped_ffn_mx")


def moe_ffn_mx_intermediate(ws, T: int, H: int, I: int, top_k: int):
    """(codes [T*top_k, Ip] uint8, scale bytes [G, T*top_k, 16] uint8 with
    G = ceil(Ip/512): chunk c of row r at [c // 16, r, c % 16]) views of the
    MX intermediate held in an MX FFN workspace, rows in expert order."""
    c, sc = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib().moe_ffn_mx_intermediate(_p(ws), T, H, I, top_k, ctypes.byref(c), ctypes.byref(sc)),
           "moe_ffn_mx_intermediate")
    Ip = (I + 127) // 128 * 128
    base = ws.data_ptr()
    oc, osc = c.value - base, sc.value - base
    P = T * top_k
    G = (Ip + 511) // 512
    return ws[oc: oc + P * Ip].view(P, Ip), ws[osc: osc + G * P * 16].view(G, P, 16)


def moe_debug_grouped_down_mx(h_codes, h_scales, topk_w, expert_offsets, sorted_pairs, w_down, s_down, y, ws,
                              stream=None):
    """Test hook: the MX down GEMM alone on a caller-supplied intermediate
    (h_codes [T*top_k, Ip] uint8, h_scales [G, T*top_k, 16] uint8 as
    moe_ffn_mx_intermediate lays it out, expert order), writing y
    [T, top_k, H] for the valid pairs."""
    T, k = topk_w.shape
    E, H, I = w_down.shape
    _check(lib().moe_debug_grouped_down_mx(_p(h_codes), _p(h_scales), T, H, k, _p(topk_w), _p(expert_offsets),
                                           _p(sorted_pairs), E, I, _p(w_down), _p(s_down), _p(y), _p(ws),
                                           ws.numel(), _s(stream)), "moe_debug_grouped_down_mx")


def moe_combine(y, topk_ids, num_experts, routed_scaling, out_f32, out_bf16, ws, stream=None):
    T, top_k = topk_ids.shape
    H = out_f32.shape[1]
    _check(lib().moe_combine(_p(y), _p(topk_ids), T, H, top_k, num_experts, float(routed_scaling),
                             _p(out_f32), _p(out_bf16), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "moe_combine")


def moe_get_device_status(ws) -> int:
    v = ctypes.c_int(0)
    _check(lib().moe_get_device_status(_p(ws), ctypes.byref(v)), "moe_get_device_status")
    return int(v.value)


def moe_debug_encode(inp, out, stream=None):
    _check(lib().moe_debug_encode(_p(inp), inp.numel(), _p(out), _s(stream)), "moe_debug_encode")


def moe_ffn_intermediate(ws, T: int, H: int, I: int, top_k: int):
    """(codes [T*top_k, Ip] uint8, scales [T*top_k, ceil(I/128)] float32)
    views of the intermediate held in a grouped-FFN workspace, rows in
    expert order."""
    c, sc = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib().moe_ffn_intermediate(_p(ws), T, H, I, top_k, ctypes.byref(c), ctypes.byref(sc)),
           "moe_ffn_intermediate")
    GI = (I + 127) // 128
    base = ws.data_ptr()
    oc, osc = c.value - base, sc.value - base
    P = T * top_k
    codes = ws[oc: oc + P * GI * 128].view(P, GI * 128)
    scales = ws[osc: osc + P * GI * 4].view(torch.float32).view(P, GI)
    return codes, scales


def moe_debug_grouped_down(h_codes, h_scales, topk_w, expert_offsets, sorted_pairs, w_down, s_down, y, ws,
                           stream=None):
    """Test hook: the down GEMM alone on a caller-supplied intermediate
    (h_codes [T*top_k, Ip] uint8, h_scales [T*top_k, ceil(I/128)] float32,
    rows in expert order), writing y [T, top_k, H] for the valid pairs."""
    T, k = topk_w.shape
    E, H, I = w_down.shape
    _check(lib().moe_debug_grouped_down(_p(h_codes), _p(h_scales), T, H, k, _p(topk_w), _p(expert_offsets),
                                        _p(sorted_pairs), E, I, _p(w_down), _p(s_down), _p(y), _p(ws),
                                        ws.numel(), _s(stream)), "moe_debug_grouped_down")


def moe_layer_workspace_bytes(T: int, H: int, I: int, E: int, top_k: int) -> int:
    return int(lib().moe_layer_workspace_bytes(T, H, I, E, top_k))


def moe_layer(logits, x, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling, out_f32, out_bf16, ws,
              stream=None):
    """The whole layer (moe_route_quant, moe_grouped_ffn, moe_combine) over
    one workspace of moe_layer_workspace_bytes."""
    T, E = logits.shape
    H = x.shape[1]
    I = w_gate.shape[1]
    _check(lib().moe_layer(_p(logits), _p(x), T, H, E, top_k, I, _p(w_gate), _p(s_gate), _p(w_up), _p(s_up),
                           _p(w_down), _p(s_down), routed_scaling, _p(out_f32), _p(out_bf16), _p(ws),
                           ws.numel() * ws.element_size(), _s(stream)), "moe_layer")


def moe_layer_get_device_status(ws, T: int, H: int, I: int, E: int, top_k: int) -> int:
    v = ctypes.c_int(0)
    _check(lib().moe_layer_get_device_status(_p(ws), T, H, I, E, top_k, ctypes.byref(v)),
           "moe_layer_get_device_status")
    return v.value


class LayerPlan:
    """The layer captured into a CUDA graph for fixed buffers (the C ABI's
    moe_layer_plan).  ``x`` and ``logits`` are the input buffers the graph
    reads and ``out`` the FP32 rows it writes; copy each batch into ``x`` and
    ``logits`` before ``launch``.  The plan owns its workspace."""

    def __init__(self, x, logits, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling,
                 out_bf16=None, stage_events=None, fused_combine: bool = False):
        T, E = logits.shape
        H = x.shape[1]
        I = w_gate.shape[1]
        self.shape = (T, H, I, E, int(top_k))
        self.x, self.logits = x, logits
        self.w = (w_gate, s_gate, w_up, s_up, w_down, s_down)
        self.out = torch.empty((T, H), dtype=torch.float32, device=x.device)
        self.out_bf16 = out_bf16
        self.ws = torch.empty((moe_layer_workspace_bytes(T, H, I, E, top_k),), dtype=torch.uint8, device=x.device)
        self.events = stage_events
        evs = None
        if stage_events is not None:
            assert len(stage_events) == 6
            for e in stage_events:
                if not e.cuda_event:  # torch creates the CUDA event at its first record
                    e.record()
            evs = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in stage_events])
        h = ctypes.c_void_p(0)
        _check(lib().moe_layer_plan_create_ex(ctypes.byref(h), _p(logits), _p(x), T, H, E, int(top_k), I,
                                              *[_p(t) for t in self.w], float(routed_scaling), _p(self.out),
                                              _p(out_bf16), _p(self.ws), self.ws.numel(), evs,
                                              1 if fused_combine else 0), "moe_layer_plan_create")
        self._h = h

    def launch(self, stream=None) -> torch.Tensor:
        _check(lib().moe_layer_plan_launch(self._h, _s(stream)), "moe_layer_plan_launch")
        return self.out

    def device_status(self) -> int:
        return moe_layer_get_device_status(self.ws, *self.shape)

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().moe_layer_plan_destroy(self._h)
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_grouped_ffn_combine(codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs, w_gate, s_gate,
                            w_up, s_up, w_down, s_down, y, routed_scaling, out_f32, out_bf16, ws, stream=None,
                            stage_events=None):
    """moe_grouped_ffn with the combine fused into the down GEMM: writes
    out_f32 (and out_bf16) as moe_combine would, bit for bit."""
    T, H = codes.shape
    k = topk_ids.shape[1]
    E, I = w_gate.shape[0], w_gate.shape[1]
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * 4)(*[e.cuda_event for e in stage_events])
    _check(lib().moe_grouped_ffn_combine(_p(codes), _p(act_scales), T, H, _p(topk_ids), _p(topk_w), k,
                                         _p(expert_offsets), _p(sorted_pairs), E, I, _p(w_gate), _p(s_gate),
                                         _p(w_up), _p(s_up), _p(w_down), _p(s_down), _p(y), routed_scaling,
                                         _p(out_f32), _p(out_bf16), _p(ws), ws.numel() * ws.element_size(),
                                         _s(stream), ev), "moe_grouped_ffn_combine")


def moe_route_shared(logits, top_k, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, stream=None):
    """moe_route plus the shared-expert slot: topk_ids / topk_w [T, top_k+1]
    with slot top_k = (E, 1.0); sorted_pairs [T*(top_k+1)] (routed pairs)."""
    T, E = logits.shape
    _check(lib().moe_route_shared(_p(logits), T, E, top_k, _p(topk_ids), _p(topk_w), _p(expert_offsets),
                                  _p(sorted_pairs), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "moe_route_shared")


def moe_combine_shared(y, topk_ids, num_experts, routed_scaling, out_f32, out_bf16, ws, stream=None):
    """moe_combine with the shared-expert slot (id num_experts) added after
    the routed scaling."""
    T, k, H = y.shape
    _check(lib().moe_combine_shared(_p(y), _p(topk_ids), T, H, k, num_experts, routed_scaling, _p(out_f32),
                                    _p(out_bf16), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "moe_combine_shared")


def moe_ep_plan_workspace_bytes(T: int, top_k: int, world: int) -> int:
    return int(lib().moe_ep_plan_workspace_bytes(T, top_k, world))


def moe_ep_plan(topk_ids, num_experts, world, rank, T_home, local_ids, send_rows, recv_rows, offs_oh, offs_ho, ws,
                stream=None):
    T, k = topk_ids.shape
    _check(lib().moe_ep_plan(_p(topk_ids), T, k, num_experts, world, rank, T_home, _p(local_ids), _p(send_rows),
                             _p(recv_rows), _p(offs_oh), _p(offs_ho), _p(ws), ws.numel() * ws.element_size(),
                             _s(stream)), "moe_ep_plan")


def moe_permute(ids, num_experts, expert_offsets, sorted_pairs, ws, stream=None):
    """The stable permutation of moe_route on caller-given ids [T, k]."""
    T, k = ids.shape
    _check(lib().moe_permute(_p(ids), T, num_experts, k, _p(expert_offsets), _p(sorted_pairs), _p(ws),
                             ws.numel() * ws.element_size(), _s(stream)), "moe_permute")


def moe_grouped_ffn_rows(codes, act_scales, topk_ids, topk_w, expert_offsets, sorted_pairs, w_gate, s_gate, w_up,
                         s_up, w_down, s_down, y, y_rows, ws, stream=None):
    """moe_grouped_ffn writing pair p to row y_rows[p] of y (-1: not written)."""
    T, H = codes.shape
    k = topk_ids.shape[1]
    E, I = w_gate.shape[0], w_gate.shape[1]
    _check(lib().moe_grouped_ffn_rows(_p(codes), _p(act_scales), T, H, _p(topk_ids), _p(topk_w), k,
                                      _p(expert_offsets), _p(sorted_pairs), E, I, _p(w_gate), _p(s_gate), _p(w_up),
                                      _p(s_up), _p(w_down), _p(s_down), _p(y), _p(y_rows), y.shape[0], _p(ws),
                                      ws.numel() * ws.element_size(), _s(stream), None), "moe_grouped_ffn_rows")


def moe_combine_rows(y, rows, routed_scaling, out_f32, out_bf16, ws, stream=None):
    """out[t] = routed_scaling * sum_j y[rows[t, j]] over rows >= 0, slot order."""
    T, k = rows.shape
    H = out_f32.shape[1]
    _check(lib().moe_combine_rows(_p(y), y.shape[0], _p(rows), T, H, k, routed_scaling, _p(out_f32), _p(out_bf16),
                                  _p(ws), ws.numel() * ws.element_size(), _s(stream)), "moe_combine_rows")


# ------------------------------------------------------------------ layer

class RoutedMoE:
    """One routed-expert layer: resident FP8 weights and their block scales,
    plus output and workspace buffers sized for up to `max_tokens` rows.
    ``forward`` enqueues moe_route_quant (or, with fused=False, moe_quant_act
    and moe_route), moe_grouped_ffn and moe_combine on the current stream
    and returns the FP32 output rows."""

    def __init__(self, w_gate, s_gate, w_up, s_up, w_down, s_down, top_k: int, routed_scaling: float,
                 max_tokens: int):
        self.w = (w_gate, s_gate, w_up, s_up, w_down, s_down)
        self.E, self.I, self.H = w_gate.shape
        self.k = int(top_k)
        self.rs = float(routed_scaling)
        self.max_tokens = int(max_tokens)
        dev = w_gate.device
        T, H, E, k = self.max_tokens, self.H, self.E, self.k
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        self.codes = torch.empty((T, H), dtype=u8, device=dev)
        self.scales = torch.empty((T, H // 128), dtype=f32, device=dev)
        self.ids = torch.empty((T, k), dtype=i32, device=dev)
        self.tw = torch.empty((T, k), dtype=f32, device=dev)
        self.offsets = torch.empty((E + 1,), dtype=i32, device=dev)
        self.sorted = torch.empty((T * k,), dtype=i32, device=dev)
        self.y = torch.empty((T, k, H), dtype=f32, device=dev)
        self.out = torch.empty((T, H), dtype=f32, device=dev)
        self.ws_route = torch.empty((moe_route_workspace_bytes(T, E, k),), dtype=u8, device=dev)
        self.ws_ffn = torch.empty((moe_ffn_workspace_bytes(T, H, self.I, E, k),), dtype=u8, device=dev)
        self.ws_comb = torch.empty((moe_combine_workspace_bytes(),), dtype=u8, device=dev)

    def forward(self, x: torch.Tensor, logits: torch.Tensor, out_bf16: torch.Tensor | None = None,
                stream=None, stage_events=None, fused: bool = True) -> torch.Tensor:
        """stage_events: None, or 7 recorded torch.cuda.Events marking the
        start of quantise, route, gather, gate/up, down, combine and the end
        (fused: the first two both mark the start of moe_route_quant)."""
        T = x.shape[0]
        assert T <= self.max_tokens and x.shape[1] == self.H and logits.shape == (T, self.E)
        codes, scales = self.codes[:T], self.scales[:T]
        ids, tw, srt = self.ids[:T], self.tw[:T], self.sorted[: T * self.k]
        y, out = self.y[:T], self.out[:T]
        ev = stage_events
        s = torch.cuda.current_stream() if stream is None else stream
        if ev is not None:
            ev[0].record(s)
        if fused:
            if ev is not None:
                ev[1].record(s)
            moe_route_quant(logits, x, self.k, ids, tw, self.offsets, srt, codes, scales, self.ws_route, stream)
        else:
            moe_quant_act(x, codes, scales, stream)
            if ev is not None:
                ev[1].record(s)
            moe_route(logits, self.k, ids, tw, self.offsets, srt, self.ws_route, stream)
        moe_grouped_ffn(codes, scales, ids, tw, self.offsets, srt, *self.w, y, self.ws_ffn, stream,
                        stage_events=None if ev is None else ev[2:6])
        moe_combine(y, ids, self.E, self.rs, out, out_bf16, self.ws_comb, stream)
        if ev is not None:
            ev[6].record(s)
        return out

    def device_status(self) -> int:
        return (moe_get_device_status(self.ws_route) | moe_get_device_status(self.ws_ffn)
                | moe_get_device_status(self.ws_comb))


class RoutedMoEMX:
    """One routed-expert layer of the MXFP8 variant: resident E4M3 weights
    with UE8M0 scales per 32 values (packed once by moe_mx_pack_scales at
    construction), buffers for up to `max_tokens` rows.  ``forward`` enqueues
    moe_quant_act_mx, moe_route, moe_grouped_ffn_mx and moe_combine on the
    current stream and returns the FP32 output rows."""

    def __init__(self, w_gate, s_gate, w_up, s_up, w_down, s_down, top_k: int, routed_scaling: float,
                 max_tokens: int):
        self.E, self.I, self.H = w_gate.shape
        self.w = (w_gate, moe_mx_pack_scales(s_gate), w_up, moe_mx_pack_scales(s_up), w_down,
                  moe_mx_pack_scales(s_down))
        self.k = int(top_k)
        self.rs = float(routed_scaling)
        self.max_tokens = int(max_tokens)
        dev = w_gate.device
        T, H, E, k = self.max_tokens, self.H, self.E, self.k
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        self.codes = torch.empty((T, H), dtype=u8, device=dev)
        self.scales = torch.empty((T, H // 32), dtype=u8, device=dev)
        self.ids = torch.empty((T, k), dtype=i32, device=dev)
        self.tw = torch.empty((T, k), dtype=f32, device=dev)
        self.offsets = torch.empty((E + 1,), dtype=i32, device=dev)
        self.sorted = torch.empty((max(T * k, 1),), dtype=i32, device=dev)
        self.y = torch.empty((T, k, H), dtype=f32, device=dev)
        self.out = torch.empty((T, H), dtype=f32, device=dev)
        self.ws_route = torch.empty((moe_route_workspace_bytes(T, E, k),), dtype=u8, device=dev)
        self.ws_ffn = torch.empty((moe_ffn_mx_workspace_bytes(T, H, self.I, E, k),), dtype=u8, device=dev)
        self.ws_comb = torch.empty((moe_combine_workspace_bytes(),), dtype=u8, device=dev)

    def forward(self, x: torch.Tensor, logits: torch.Tensor, out_bf16: torch.Tensor | None = None,
                stream=None, stage_events=None) -> torch.Tensor:
        """stage_events: None, or 6 recorded torch.cuda.Events marking the
        start of quantise + route, gather, gate/up, down, combine and the end."""
        T = x.shape[0]
        assert T <= self.max_tokens and x.shape[1] == self.H and logits.shape == (T, self.E)
        codes, scales = self.codes[:T], self.scales[:T]
        ids, tw, srt = self.ids[:T], self.tw[:T], self.sorted[: max(T * self.k, 1)]
        y, out = self.y[:T], self.out[:T]
        ev = stage_events
        s = torch.cuda.current_stream() if stream is None else stream
        if ev is not None:
            ev[0].record(s)
        moe_quant_act_mx(x, codes, scales, stream)
        moe_route(logits, self.k, ids, tw, self.offsets, srt, self.ws_route, stream)
        moe_grouped_ffn_mx(codes, scales, ids, tw, self.offsets, srt, *self.w, y, self.ws_ffn, stream,
                           stage_events=None if ev is None else ev[1:5])
        moe_combine(y, ids, self.E, self.rs, out, out_bf16, self.ws_comb, stream)
        if ev is not None:
            ev[5].record(s)
        return out

    def device_status(self) -> int:
        return (moe_get_device_status(self.ws_route) | moe_get_device_status(self.ws_ffn)
                | moe_get_device_status(self.ws_comb))


