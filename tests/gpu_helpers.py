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


_ref_cache: dict = {}


def oracle_layer_h(wl: mi.Workload, h: dict, seed: int = 0, tokens=None):
    """oracle_layer(..., want_h=True) for the workload's inputs of ``seed``,
    kept for the other tests of the same inputs (the oracle is the slow
    side)."""
    key = (wl, seed, None if tokens is None else np.asarray(tokens).tobytes())
    if key not in _ref_cache:
        if len(_ref_cache) > 3:
            _ref_cache.clear()
        _ref_cache[key] = oracle_layer(wl, h, tokens=tokens, want_h=True)
    return _ref_cache[key]


# ----------------------------------------------------------------------------
# Intermediate requantisation: a floating-point decision of an integer code.
# The CUDA path decides from FP32 tensor-core sums, the oracle from FP64 sums
# rounded to FP32; where the exact value lies within the FP32 error of an E4M3
# rounding boundary both codes are valid.  The comparison takes the oracle's
# codes as the reference and accepts a differing GPU code only if it is the
# adjacent code across a boundary that lies within a bound DERIVED from the
# operands (below) of the oracle's own quotient; the output tolerance of the
# affected elements widens by exactly the effect of those codes.  The GPU's
# intermediate scales must lie within the same derived bound of the
# oracle's.  No GPU value is ever fed to the oracle.
#
# The bound, per intermediate element (pair r, column n), with u = 2^-24:
#   g = sum_kb c_kb P_kb, c_kb = fl(sa*sw), P_kb the tensor core's sum of the
#   128 exact E4M3 products of K block kb, folded by one FMA per block:
#     |g_gpu - g| <= (gamma_127(2u) + gamma_(nkb+1)(u)) * S_g,
#   S_g = sum_k |sa*sw*dec(a_k)*dec(w_k)| (the same dot with absolute
#   values), gamma_m(v) = m v / (1 - m v).  The tensor core's additions are
#   taken as faithful (error < 1 ulp, 2u relative), which covers rounding
#   to nearest and toward zero in any order.  Same for u.
#   SiLU on the GPU: e = ex2.approx(fl(-g log2 e)), r = rcp.approx(fl(1+e)),
#   fl(g r): relative error <= 2u|g| (the rounded exponent argument)
#   + EPS_EX2 + EPS_RCP + 2u, with the PTX ISA's stated accuracies of
#   ex2.approx.f32 (2^-22 relative) and rcp.approx.f32 (1 ulp, 2^-23).
#   |dSiLU/dg| <= 1.1 everywhere, so
#     e_h = 1.1 E_g |u| + |SiLU(g)| E_u + 1.1 E_g E_u
#           + (|SiLU(g)| + 1.1 E_g)(|u| + E_u)(eps_silu + u) + u|h|
#   bounds |h_gpu - h32| (h32 = the oracle's FP32 h).
#   Quotients: the GPU's fl(h_gpu * rcp_rn(s_gpu)), the oracle's
#   fl(h32 / s_o):
#     |q_gpu - q_o| <= e_h / s_gpu + |q_o| |s_o / s_gpu - 1| + 4u |q_o|.
#   A flip is accepted iff the rounding boundary between the two codes lies
#   within that distance of q_o.  Scales: |amax_gpu - amax_o| <= max e_h over
#   the group, so |s_gpu - s_o| <= max e_h / 448 + u (s_gpu + s_o).

U32 = 2.0 ** -24
EPS_EX2 = 2.0 ** -22
EPS_RCP = 2.0 ** -23

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


def _gamma(m: int, v: float) -> float:
    return m * v / (1.0 - m * v)


def _dequant_rows(codes_u8: np.ndarray, scales: np.ndarray) -> torch.Tensor:
    """[n, K] codes with [n, K/128] scales -> float64 [n, K] values."""
    dec = torch.from_numpy(_dec())
    v = dec[torch.from_numpy(np.ascontiguousarray(codes_u8)).long()]
    sc = torch.from_numpy(np.ascontiguousarray(scales)).double().repeat_interleave(128, dim=1)[:, : v.shape[1]]
    return v * sc


def _dequant_weight(w_u8: torch.Tensor, s: torch.Tensor, rows: int, cols: int) -> torch.Tensor:
    """One expert's [rows, cols] codes with its [ceil(rows/128), cols/128]
    block scales -> float64 values."""
    dec = torch.from_numpy(_dec())
    v = dec[w_u8.long()]
    sc = s.double().repeat_interleave(128, dim=0).repeat_interleave(128, dim=1)[:rows, :cols]
    return v * sc


def intermediate_error_bound(wl, h: dict, act_codes, act_scales, ids, toks):
    """Per-element bound e_h [n, k, I] on |h_gpu - h32| (the derivation
    above), from the operands of the selected tokens ``toks`` (ids [n, k])."""
    H, I = wl.H, wl.I
    nkb = H // 128
    cg = (_gamma(127, 2 * U32) + _gamma(nkb + 1, U32)) * 1.0001
    A = _dequant_rows(np.asarray(act_codes)[toks], np.asarray(act_scales)[toks])  # [n, H]
    Aabs = A.abs()
    n, k = ids.shape
    eh = np.zeros((n, k, I), np.float64)
    wg, sg, wu, su = (torch.as_tensor(h[key]) for key in ("w_gate", "s_gate", "w_up", "s_up"))
    for e in np.unique(ids[ids >= 0]):
        ti, ji = np.nonzero(ids == e)
        a, aa = A[ti], Aabs[ti]
        Wg = _dequant_weight(wg[e], sg[e], I, H)
        Wu = _dequant_weight(wu[e], su[e], I, H)
        g, u = (a @ Wg.T).numpy(), (a @ Wu.T).numpy()
        Eg, Eu = cg * (aa @ Wg.abs().T).numpy(), cg * (aa @ Wu.abs().T).numpy()
        sig = 1.0 / (1.0 + np.exp(-np.clip(g, -700, 700)))
        silu = np.abs(g * sig)
        eps_silu = 2 * U32 * (np.abs(g) + Eg) + EPS_EX2 + EPS_RCP + 2 * U32
        au = np.abs(u)
        e = (1.1 * Eg * au + silu * Eu + 1.1 * Eg * Eu
             + (silu + 1.1 * Eg) * (au + Eu) * (eps_silu + U32) * 1.0001 + U32 * silu * au * 1.0001)
        eh[ti, ji] = e
    return eh


def check_layer(wl, layer, gpu_out, ref, h, tokens=None):
    """Full comparison of a layer call with the oracle (``ref`` computed with
    want_h=True for ``tokens``, default all).  Returns a dict of statistics;
    ``plain_out_of_tol`` counts the outputs beyond the method's literal
    tolerance (each must be explained by accepted intermediate flips)."""
    T = gpu_out.shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    g_out = gpu_out.detach().double().cpu().numpy()[toks]
    gc, gs = gpu_intermediate_by_pair(layer, T)
    gc, gs = gc[toks], gs[toks]
    ids = np.asarray(ref["ids"])
    if ids.shape[0] != toks.size:
        ids = ids[toks]
    w = np.asarray(ref["w"])
    if w.shape[0] != toks.size:
        w = w[toks]
    oc, ohf, osc = ref["h_codes"], ref["h_fp32"], ref["h_scales"]
    I = wl.I
    valid = ids >= 0                                   # [n, k]
    assert np.all(gc[..., I:][valid] == 0), "padding columns of the intermediate must be zero"
    eh = intermediate_error_bound(wl, h, ref["codes"], ref["scales"], ids, toks)   # [n, k, I]
    stats = {"codes": int(valid.sum()) * I}

    # scales: every finite group of a valid pair within the derived bound
    GI = wl.GI
    ehp = np.zeros(eh.shape[:2] + (GI * 128,))
    ehp[..., :I] = eh
    eh_grp = ehp.reshape(eh.shape[:2] + (GI, 128)).max(axis=-1)           # [n, k, GI]
    vs = valid[..., None] & np.isfinite(osc)
    hp = np.zeros(ohf.shape[:2] + (GI * 128,), np.float64)
    hp[..., : ohf.shape[2]] = np.abs(ohf.astype(np.float64))
    amax_o = hp.reshape(ohf.shape[:2] + (GI, 128)).max(axis=-1)
    vs &= amax_o > 0                                   # s = 1 by rule for all-zero groups
    s_lim = eh_grp / 448.0 * (1 + U32) + U32 * (np.abs(gs.astype(np.float64)) + np.abs(osc.astype(np.float64)))
    sdiff = np.abs(gs.astype(np.float64) - osc.astype(np.float64))
    assert np.all(sdiff[vs] <= s_lim[vs]), (
        f"intermediate scale beyond its derived bound: worst {(sdiff[vs] / s_lim[vs]).max():.3g}x")
    stats["max_scale_over_bound"] = float((sdiff[vs] / s_lim[vs]).max(initial=0.0))

    flips = (gc != oc) & valid[..., None]
    flips[..., I:] = False
    n_flip = int(flips.sum())
    stats.update(flips=n_flip, flip_rate=n_flip / max(stats["codes"], 1), max_flip_over_bound=0.0)
    rank = _value_rank()
    dec = _dec()
    allowance = np.zeros_like(g_out)
    if n_flip:
        t_i, j_i, c_i = np.nonzero(flips)
        r_g = rank[gc[t_i, j_i, c_i]]
        r_o = rank[oc[t_i, j_i, c_i]]
        # rank 0: the same value with the other sign of zero; rank 1: the
        # neighbouring code across one rounding boundary
        assert np.all(np.abs(r_g - r_o) <= 1), "a differing intermediate code is not adjacent"
        s_o = osc[t_i, j_i, c_i // 128].astype(np.float64)
        s_g = gs[t_i, j_i, c_i // 128].astype(np.float64)
        q_o = (ohf[t_i, j_i, c_i].astype(np.float32) / s_o.astype(np.float32)).astype(np.float64)
        mid = (dec[gc[t_i, j_i, c_i]] + dec[oc[t_i, j_i, c_i]]) / 2
        dist = np.abs(q_o - mid)
        lim = eh[t_i, j_i, c_i] / s_g + np.abs(q_o) * np.abs(s_o / s_g - 1.0) + 4 * U32 * np.abs(q_o)
        stats["max_flip_over_bound"] = float((dist / lim).max())
        assert np.all(dist <= lim), (
            f"a differing code is {(dist / lim).max():.3g}x its derived distance from the rounding boundary")
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
    # every element beyond the literal tolerance must be explained by flips
    assert np.all(allowance[plain_bad] > 0)
    stats["median_tok_rel"] = float(np.median(tok_rel(g_out, r_out))) if err.size else 0.0
    return stats


def check_down_on_oracle_intermediate(wl, layer, ref, h, tokens=None):
    """Diagnostic of the down projection and the combine alone: the ORACLE's
    intermediate codes and scales (want_h=True) are fed to the CUDA down GEMM
    (moe_debug_grouped_down) and the CUDA combine, so both sides start from
    the same intermediate and no requantisation decision can differ.  The
    result must meet the method's literal tolerance on every element of the
    selected tokens, with no allowance.  Routing and the permutation were
    checked bit-exact against the oracle's before this is called."""
    k = layer.k
    T = np.asarray(ref["ids"]).shape[0]  # the oracle routes every token of the call
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    Ip, GI = wl.Ip, wl.GI
    hc = np.zeros((T, k, Ip), np.uint8)
    hs = np.ones((T, k, GI), np.float32)
    hc[toks], hs[toks] = ref["h_codes"], ref["h_scales"]
    sp = ref["sorted_pairs"]
    P = int(ref["offsets"][-1])
    hc_sorted = np.zeros((T * k, Ip), np.uint8)
    hs_sorted = np.ones((T * k, GI), np.float32)
    hc_sorted[:P] = hc.reshape(T * k, Ip)[sp[:P]]
    hs_sorted[:P] = hs.reshape(T * k, GI)[sp[:P]]
    dev = layer.ids.device
    y = torch.zeros((T, k, wl.H), dtype=torch.float32, device=dev)
    ws = torch.zeros((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device=dev)
    assert np.array_equal(layer.offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(layer.sorted[:P].cpu().numpy(), sp[:P])
    fm.moe_debug_grouped_down(torch.from_numpy(hc_sorted).to(dev), torch.from_numpy(hs_sorted).to(dev),
                              layer.tw[:T], layer.offsets, layer.sorted[: T * k], layer.w[4], layer.w[5], y, ws)
    assert fm.moe_get_device_status(ws) == 0
    out = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    fm.moe_combine(y, layer.ids[:T], wl.E, wl.routed_scaling, out, None, ws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    g = out.double().cpu().numpy()[toks]
    r = np.asarray(ref["out"])
    tol = REL_TOL * np.abs(r).max(axis=1, keepdims=True) + ABS_TOL
    err = np.abs(g - r)
    worst = float((err / tol).max()) if err.size else 0.0
    assert not (err > tol).any(), f"{int((err > tol).sum())} outputs beyond the literal tolerance; worst {worst:.3f}"
    return {"worst_err_over_tol": worst, "elements": int(err.size)}
