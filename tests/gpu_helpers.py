"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI binding and the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import hashlib

import numpy as np
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle

# Output tolerance of the method's statement: |err| <= 2e-3 * ||row||_inf + 1e-3.
REL_TOL = 2e-3
ABS_TOL = 1e-3

_cache: dict = {}


def inputs(wl: mi.Workload, seed: int = 0, T: int | None = None):
    """CUDA tensors of a workload and CPU copies of the same bytes."""
    key = (wl, seed, T)
    if key not in _cache:
        if len(_cache) > 2:
            _cache.clear()
            torch.cuda.empty_cache()
        d = mi.make_inputs(wl, seed, "cuda", T=T)
        h = {k: v.cpu() for k, v in d.items()}
        _cache[key] = (d, h)
    return _cache[key]


def run_layer(wl: mi.Workload, d: dict, routed_scaling: float | None = None, bf16: bool = False):
    rs = wl.routed_scaling if routed_scaling is None else routed_scaling
    T = d["x"].shape[0]
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"],
                         wl.k, rs, max_tokens=max(T, 1))
    ob = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda") if bf16 else None
    out = layer.forward(d["x"], d["logits"], out_bf16=ob)
    torch.cuda.synchronize()
    return layer, out, ob


def assert_close_rows(gpu_out, ref_out, rows=None):
    g = gpu_out.detach().double().cpu().numpy() if hasattr(gpu_out, "detach") else np.asarray(gpu_out)
    if rows is not None:
        g = g[rows]
    ref = np.asarray(ref_out)
    tol = REL_TOL * np.abs(ref).max(axis=1, keepdims=True) + ABS_TOL
    err = np.abs(g - ref)
    bad = err > tol
    assert not bad.any(), (
        f"{int(bad.sum())} of {bad.size} outputs out of tolerance; worst err {err.max():.3e}, "
        f"worst err/tol {(err / tol).max():.3f}")
    return err, tol


def tok_rel(gpu_out, ref_out):
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    return np.linalg.norm(g - r, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-300)


def sha(t: torch.Tensor) -> str:
    return hashlib.sha256(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()).hexdigest()


def oracle_layer(wl: mi.Workload, h: dict, tokens=None, routed_scaling=None, **kw):
    rs = wl.routed_scaling if routed_scaling is None else routed_scaling
    return oracle.moe_layer(h["x"], h["logits"], wl.k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"],
                            h["w_down"], h["s_down"], rs, tokens=tokens, **kw)


# ----------------------------------------------------------------------------
# Intermediate requantisation: a floating-point decision of an integer code.
# The CUDA path decides from FP32 tensor-core sums, the oracle from FP64 sums
# rounded to FP32; where the exact value lies within the FP32 error of an E4M3
# rounding boundary both codes are valid.  The comparison below takes the
# oracle's codes as the reference, accepts a differing GPU code only if it is
# the adjacent code across a boundary the oracle's own value sits next to,
# and widens the output tolerance of the affected elements by exactly the
# bounded effect of those codes.  No GPU value is ever fed to the oracle.

_DEC = None


def _dec():
    global _DEC
    if _DEC is None:
        _DEC = oracle.e4m3_decode_all()
    return _DEC


def _value_rank():
    """Rank of each code's value in the ordered set of E4M3 values (+0 and -0
    share a rank)."""
    vals = _dec()
    uniq = np.unique(vals)  # -0.0 == 0.0 collapse
    return np.searchsorted(uniq, vals)


def gpu_intermediate_by_pair(layer, T: int):
    """GPU intermediate codes/scales regrouped to [T, k, Ip] / [T, k, GI]."""
    k, I, H = layer.k, layer.I, layer.H
    codes, scales = fm.moe_ffn_intermediate(layer.ws_ffn, T, H, I, k)
    P = int(layer.offsets[-1].item())
    sp = layer.sorted[:P].cpu().numpy()
    Ip = codes.shape[1]
    GI = scales.shape[1]
    gc = np.zeros((T * k, Ip), np.uint8)
    gs = np.zeros((T * k, GI), np.float32)
    gc[sp] = codes[:P].cpu().numpy()
    gs[sp] = scales[:P].cpu().numpy()
    return gc.reshape(T, k, Ip), gs.reshape(T, k, GI)


def check_layer(wl, layer, gpu_out, ref, h, tokens=None, mid_tol=1e-4):
    """Full comparison of a layer call with the oracle (``ref`` computed with
    want_h=True for ``tokens``, default all).  Returns a dict of statistics."""
    T = gpu_out.shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    g_out = gpu_out.detach().double().cpu().numpy()[toks]
    gc, gs = gpu_intermediate_by_pair(layer, T)
    gc, gs = gc[toks], gs[toks]
    ids = ref["ids"] if tokens is None else ref["ids"]
    ids = np.asarray(ids)
    if ids.shape[0] != toks.size:
        ids = ids[toks]
    w = np.asarray(ref["w"])
    if w.shape[0] != toks.size:
        w = w[toks]
    oc, ohf, osc = ref["h_codes"], ref["h_fp32"], ref["h_scales"]
    valid = ids >= 0                                   # [n, k]
    flips = (gc != oc) & valid[..., None]
    flips[..., wl.I:] = False                          # padding columns are compared below
    assert np.all(gc[..., wl.I:][valid] == 0), "padding columns of the intermediate must be zero"
    n_valid_codes = int(valid.sum()) * wl.I
    n_flip = int(flips.sum())
    rank = _value_rank()
    dec = _dec()
    stats = {"flips": n_flip, "codes": n_valid_codes, "flip_rate": n_flip / max(n_valid_codes, 1),
             "max_mid_dist": 0.0}
    vs = valid[..., None] & np.isfinite(osc) & (osc > 0)
    stats["max_scale_rel_diff"] = float(np.max(np.abs(gs[vs] / osc[vs] - 1.0), initial=0.0))
    allowance = np.zeros_like(g_out)
    if n_flip:
        t_i, j_i, c_i = np.nonzero(flips)
        r_g = rank[gc[t_i, j_i, c_i]]
        r_o = rank[oc[t_i, j_i, c_i]]
        # rank 0: the same value with the other sign of zero; rank 1: the
        # neighbouring code across one rounding boundary
        assert np.all(np.abs(r_g - r_o) <= 1), "a differing intermediate code is not adjacent"
        s_o = osc[t_i, j_i, c_i // 128].astype(np.float32)
        q_o = (ohf[t_i, j_i, c_i].astype(np.float32) / s_o).astype(np.float64)
        mid = (dec[gc[t_i, j_i, c_i]] + dec[oc[t_i, j_i, c_i]]) / 2
        dist = np.abs(q_o - mid)
        stats["max_mid_dist"] = float(dist.max())
        lim = mid_tol * np.maximum(np.abs(mid), 1.0)
        assert np.all(dist <= lim), (
            f"a differing code is {(dist / lim).max():.3g}x the allowed distance from its rounding boundary")
        wd = h["w_down"].numpy() if hasattr(h["w_down"], "numpy") else h["w_down"]
        sd = h["s_down"].numpy() if hasattr(h["s_down"], "numpy") else h["s_down"]
        for t, j, c in zip(t_i, j_i, c_i):
            e = ids[t, j]
            delta = (dec[gc[t, j, c]] - dec[oc[t, j, c]]) * float(osc[t, j, c // 128])
            col = dec[wd[e, :, c]] * np.repeat(sd[e, :, c // 128].astype(np.float64), 128)[: wl.H]
            allowance[t] += abs(wl.routed_scaling * w[t, j] * delta) * np.abs(col)
    r_out = np.asarray(ref["out"])
    tol = REL_TOL * np.abs(r_out).max(axis=1, keepdims=True) + ABS_TOL
    err = np.abs(g_out - r_out)
    plain_bad = err > tol
    stats["plain_out_of_tol"] = int(plain_bad.sum())
    stats["worst_err_over_tol"] = float((err / tol).max()) if err.size else 0.0
    bad = err > tol + 1.001 * allowance
    assert not bad.any(), (f"{int(bad.sum())} outputs outside tolerance + flip allowance; "
                           f"worst (err-allow)/tol {((err - allowance) / tol).max():.3f}; {stats}")
    # every element beyond the plain tolerance must be explained by flips
    assert np.all(allowance[plain_bad] > 0)
    stats["median_tok_rel"] = float(np.median(tok_rel(g_out, r_out))) if err.size else 0.0
    return stats
