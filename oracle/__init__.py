"""Oracle for the routed-MoE FP8 blockwise (W8A8) prefill path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's ``smoke()`` check and
the benchmark's CPU-baseline leg may import this module.  The product path
(the CUDA library and its Python binding) never imports, links or calls it,
and this module imports nothing from the product path.

The arithmetic lives in ``oracle.c`` (plain C, FP64, OpenMP over tokens);
this file compiles it on demand with gcc and exposes numpy-level wrappers.
Each wrapper names the passage of the pages it follows; the C file states
the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Strict IEEE behaviour: no fast-math, no FMA contraction, no flush to zero.
CFLAGS = ["-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile ``oracle.c`` (or another source, for planted-mistake controls
    in the tests) into a shared library with gcc.  Returns the path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def open_library(path: str) -> ctypes.CDLL:
    """Load a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode_n.argtypes = [P, i64, P]
    lib.oracle_quant_group.argtypes = [P, i32, P, P]
    lib.oracle_quant_act.argtypes = [P, i64, i64, P, P]
    lib.oracle_route.argtypes = [P, i64, i32, i32, P, P]
    lib.oracle_permute.argtypes = [P, i64, i32, i32, P, P]
    lib.oracle_moe_ffn.argtypes = [P, P, i64, i64, P, P, i32, i32, i64,
                                   P, P, P, P, P, P, ctypes.c_double,
                                   P, i64, P, P, P, P, P, P, P, i32]
    lib.oracle_num_threads.restype = i32
    lib.oracle_ue8m0_decode.restype = ctypes.c_double
    lib.oracle_ue8m0_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_mx_quant_block.argtypes = [P, i32, P, P]
    lib.oracle_mx_quant_act.argtypes = [P, i64, i64, P, P]
    lib.oracle_mx_moe_ffn.argtypes = [P, P, i64, i64, P, P, i32, i32, i64, P, P, P, P, P, P, ctypes.c_double,
                                      P, i64, P, P, P, P, i32]
    return lib


_override = threading.local()


def _load():
    """The library in use: the default build, or one installed by ``using``."""
    lib = getattr(_override, "lib", None)
    if lib is not None:
        return lib
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = open_library(_LIB_PATH)
    return _lib


class using:
    """Context manager: route this module's functions through another build
    of the oracle (the tests use it to plant mistakes and check that the
    pins catch them)."""

    def __init__(self, lib: ctypes.CDLL):
        self.lib = lib

    def __enter__(self):
        self.prev = getattr(_override, "lib", None)
        _override.lib = self.lib
        return self.lib

    def __exit__(self, *exc):
        _override.lib = self.prev
        return False


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _np(a, dtype):
    """Accept numpy arrays or CPU torch tensors; return a contiguous numpy array."""
    if hasattr(a, "detach"):
        a = a.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_decode(b: int) -> float:
    """E4M3 byte -> value, by the format definition ("Exact AVX2 FP8
    arithmetic conversion avoids costly LUT gathers", "Semantics and scope")."""
    return float(_load().oracle_e4m3_decode(int(b) & 0xFF))


def e4m3_decode_all() -> np.ndarray:
    return np.array([e4m3_decode(b) for b in range(256)], dtype=np.float64)


def e4m3_encode(v: float) -> int:
    """FP32 value -> nearest finite E4M3 code, ties to even, saturating."""
    return int(_load().oracle_e4m3_encode(ctypes.c_float(float(v))))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Elementwise encode of an FP32 array (flattened)."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.zeros(v.size, np.uint8)
    _load().oracle_e4m3_encode_n(_ptr(v), v.size, _ptr(out))
    return out


def quant_group(x: np.ndarray):
    """Quantise one group of 1..128 FP32 values -> (codes uint8[n], scale float32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert 1 <= x.size <= 128
    codes = np.zeros(x.size, np.uint8)
    scale = np.zeros(1, np.float32)
    _load().oracle_quant_group(_ptr(x), x.size, _ptr(codes), _ptr(scale))
    return codes, scale[0]


def quant_act(x_bf16_bits) -> tuple[np.ndarray, np.ndarray]:
    """BF16 rows [T,H] (given as uint16 bits, or a torch bfloat16 tensor) ->
    codes uint8 [T,H], scales float32 [T,H/128]."""
    if hasattr(x_bf16_bits, "detach"):
        import torch
        x_bf16_bits = x_bf16_bits.detach().cpu().contiguous().view(torch.int16).numpy()
    x = np.ascontiguousarray(x_bf16_bits).view(np.uint16)
    T, H = x.shape
    assert H % 128 == 0
    codes = np.zeros((T, H), np.uint8)
    scales = np.zeros((T, H // 128), np.float32)
    _load().oracle_quant_act(_ptr(x), T, H, _ptr(codes), _ptr(scales))
    return codes, scales


def route(logits, top_k: int) -> tuple[np.ndarray, np.ndarray]:
    """Router logits [T,E] FP32 -> ids int32 [T,k], weights float64 [T,k]."""
    lg = _np(logits, np.float32)
    T, E = lg.shape
    ids = np.zeros((T, top_k), np.int32)
    w = np.zeros((T, top_k), np.float64)
    _load().oracle_route(_ptr(lg), T, E, top_k, _ptr(ids), _ptr(w))
    return ids, w


def permute(ids, num_experts: int) -> tuple[np.ndarray, np.ndarray]:
    """ids [T,k] -> expert_offsets int32 [E+1], sorted_pairs int32 [T*k]."""
    ids = _np(ids, np.int32)
    T, k = ids.shape
    off = np.zeros(num_experts + 1, np.int32)
    sp = np.zeros(T * k, np.int32)
    _load().oracle_permute(_ptr(ids), T, k, num_experts, _ptr(off), _ptr(sp))
    return off, sp


def moe_ffn(codes, act_scales, ids, w, w_gate, s_gate, w_up, s_up, w_down, s_down,
            routed_scaling: float, tokens=None, want_slots: bool = False,
            want_h: bool = False, h_override=None, n_threads: int = 0):
    """Expert FFN + combine for the listed tokens (all tokens by default).

    Returns a dict with ``out`` float64 [n,H] and, on request, ``slots``
    float64 [n,k,H] (w_j * o_j), ``h_codes`` uint8 [n,k,Ip], ``h_scales``
    float32 [n,k,G_I] and ``h_fp32`` float32 [n,k,Ip] (h before requantisation).  ``h_override=(codes, scales)`` in that layout replaces
    the intermediate used by the down projection.
    """
    codes = _np(codes, np.uint8)
    act_scales = _np(act_scales, np.float32)
    ids = _np(ids, np.int32)
    w = _np(w, np.float64) if not hasattr(w, "detach") else np.ascontiguousarray(
        w.detach().cpu().double().numpy())
    wg, wu, wd = _np(w_gate, np.uint8), _np(w_up, np.uint8), _np(w_down, np.uint8)
    sg, su, sd = _np(s_gate, np.float32), _np(s_up, np.float32), _np(s_down, np.float32)
    T, H = codes.shape
    k = ids.shape[1]
    E, I, _ = wg.shape
    GI = (I + 127) // 128
    Ip = GI * 128
    assert wd.shape == (E, H, I)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    n = tokens.size
    out = np.zeros((n, H), np.float64)
    slots = np.zeros((n, k, H), np.float64) if want_slots else None
    hc = np.zeros((n, k, Ip), np.uint8) if want_h else None
    hs = np.zeros((n, k, GI), np.float32) if want_h else None
    hf = np.zeros((n, k, Ip), np.float32) if want_h else None
    oc = os_ = None
    if h_override is not None:
        oc = np.ascontiguousarray(h_override[0], dtype=np.uint8)
        os_ = np.ascontiguousarray(h_override[1], dtype=np.float32)
        assert oc.shape == (n, k, Ip) and os_.shape == (n, k, GI)
    _load().oracle_moe_ffn(_ptr(codes), _ptr(act_scales), T, H, _ptr(ids), _ptr(w), k, E, I,
                           _ptr(wg), _ptr(sg), _ptr(wu), _ptr(su), _ptr(wd), _ptr(sd),
                           float(routed_scaling), _ptr(tokens), n, _ptr(out), _ptr(slots),
                           _ptr(hc), _ptr(hs), _ptr(hf), _ptr(oc), _ptr(os_), int(n_threads))
    res = {"out": out}
    if want_slots:
        res["slots"] = slots
    if want_h:
        res["h_codes"], res["h_scales"], res["h_fp32"] = hc, hs, hf
    return res


def route_shared(logits, top_k: int):
    """Routing with the shared expert as one more slot after the top-k
    ("GLM-5.3-Flash EXL3 on CUDA ...": all nine slots planned with E+1 expert
    ids, the shared id skipped by the routed kernels).  Reading: the extra
    slot k holds id E with weight 1 (the shared expert is not gated)."""
    ids, w = route(logits, top_k)
    T = ids.shape[0]
    E = int(logits.shape[1])
    ids2 = np.concatenate([ids, np.full((T, 1), E, np.int32)], axis=1)
    w2 = np.concatenate([w, np.ones((T, 1), w.dtype)], axis=1)
    return ids2, w2


def moe_layer_shared(x_bf16, logits, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down,
                     routed_scaling, shared_rows, tokens=None):
    """The layer with a shared-expert slot: the routed experts as in
    moe_layer, plus the caller's shared-expert row for each token, added
    unscaled: out[t] = routed_scaling * sum_j w_j o_j + shared[t] (the
    routed scaling applies to the routed experts only, as in the pages'
    layer, where routed scaling and the shared experts are separate parts).
    shared_rows: [T, H] (float32 or float64), the rows the caller writes into
    the shared slot."""
    res = moe_layer(x_bf16, logits, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling,
                    tokens=tokens)
    sh = np.asarray(shared_rows.detach().cpu().numpy() if hasattr(shared_rows, "detach") else shared_rows,
                    dtype=np.float64)
    if tokens is not None:
        sh = sh[np.asarray(tokens)]
    res["out"] = res["out"] + sh
    return res


def moe_layer(x_bf16, logits, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down,
              routed_scaling, tokens=None, **kw):
    """The whole path in the pages' order: quantise activations, route,
    permute, expert FFN, combine.  Returns a dict with every intermediate."""
    codes, scales = quant_act(x_bf16)
    ids, w = route(logits, top_k)
    E = _np(w_gate, np.uint8).shape[0]
    off, sp = permute(ids, E)
    res = moe_ffn(codes, scales, ids, w, w_gate, s_gate, w_up, s_up, w_down, s_down,
                  routed_scaling, tokens=tokens, **kw)
    res.update(codes=codes, scales=scales, ids=ids, w=w, offsets=off, sorted_pairs=sp)
    return res


# ---------------------------------------------------------------------------
# MXFP8 variant: E4M3 elements with one UE8M0 (power-of-two) scale per 32
# values along the contraction dimension.  The pages only name an MXFP8 MoE
# runtime as not yet qualified ("Exact AVX2 FP8 arithmetic conversion avoids
# costly LUT gathers", "Real-checkpoint measurements"); the rules M1-M3 in
# oracle.c are readings that follow the OCP Microscaling Formats v1.0.

def ue8m0_decode(x: int) -> float:
    """UE8M0 byte -> 2^(x-127); 0xFF -> NaN (reading M1)."""
    return float(_load().oracle_ue8m0_decode(int(x) & 0xFF))


def mx_quant_block(x: np.ndarray):
    """1..32 FP32 values -> (codes uint8[n], scale byte) by reading M2."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert 1 <= x.size <= 32
    codes = np.zeros(x.size, np.uint8)
    sc = np.zeros(1, np.uint8)
    _load().oracle_mx_quant_block(_ptr(x), x.size, _ptr(codes), _ptr(sc))
    return codes, int(sc[0])


def mx_quant_act(x_bf16_bits):
    """BF16 rows [T,H] -> codes uint8 [T,H], UE8M0 scales uint8 [T,H/32]."""
    if hasattr(x_bf16_bits, "detach"):
        import torch
        x_bf16_bits = x_bf16_bits.detach().cpu().contiguous().view(torch.int16).numpy()
    x = np.ascontiguousarray(x_bf16_bits).view(np.uint16)
    T, H = x.shape
    assert H % 32 == 0
    codes = np.zeros((T, H), np.uint8)
    scales = np.zeros((T, H // 32), np.uint8)
    _load().oracle_mx_quant_act(_ptr(x), T, H, _ptr(codes), _ptr(scales))
    return codes, scales


def mx_moe_ffn(codes, act_scales, ids, w, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling: float,
               tokens=None, want_h: bool = False, n_threads: int = 0):
    """Expert FFN + combine of the MXFP8 variant (reading M3).  Scales are
    UE8M0 bytes: activations [T,H/32], gate/up [E,I,H/32], down [E,H,I/32]."""
    codes = _np(codes, np.uint8)
    act_scales = _np(act_scales, np.uint8)
    ids = _np(ids, np.int32)
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float64))
    wg, wu, wd = _np(w_gate, np.uint8), _np(w_up, np.uint8), _np(w_down, np.uint8)
    sg, su, sd = _np(s_gate, np.uint8), _np(s_up, np.uint8), _np(s_down, np.uint8)
    T, H = codes.shape
    k = ids.shape[1]
    E, I, _ = wg.shape
    assert I % 32 == 0 and sg.shape == (E, I, H // 32) and sd.shape == (E, H, I // 32)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    n = tokens.size
    out = np.zeros((n, H), np.float64)
    hc = np.zeros((n, k, I), np.uint8) if want_h else None
    hs = np.zeros((n, k, I // 32), np.uint8) if want_h else None
    hf = np.zeros((n, k, I), np.float32) if want_h else None
    _load().oracle_mx_moe_ffn(_ptr(codes), _ptr(act_scales), T, H, _ptr(ids), _ptr(w), k, E, I, _ptr(wg),
                              _ptr(sg), _ptr(wu), _ptr(su), _ptr(wd), _ptr(sd), float(routed_scaling),
                              _ptr(tokens), n, _ptr(out), _ptr(hc), _ptr(hs), _ptr(hf), int(n_threads))
    res = {"out": out}
    if want_h:
        res["h_codes"], res["h_scales"], res["h_fp32"] = hc, hs, hf
    return res


def mx_moe_layer(x_bf16, logits, top_k, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling,
                 tokens=None, **kw):
    """The MXFP8 layer in the pages' order: quantise activations (M2), route,
    permute, expert FFN (M3), combine."""
    codes, scales = mx_quant_act(x_bf16)
    ids, w = route(logits, top_k)
    E = _np(w_gate, np.uint8).shape[0]
    off, sp = permute(ids, E)
    res = mx_moe_ffn(codes, scales, ids, w, w_gate, s_gate, w_up, s_up, w_down, s_down, routed_scaling,
                     tokens=tokens, **kw)
    res.update(codes=codes, scales=scales, ids=ids, w=w, offsets=off, sorted_pairs=sp)
    return res
