"""Checks of the MXFP8 variant's CUDA layer against the oracle (readings
M1-M3), shared by the GPU parity tests and the CPU tests of the checks
themselves: a GPU intermediate decision is accepted only inside a bound
derived from the operands; no GPU value is ever fed to the oracle."""
import numpy as np
import torch

import fp8_blockwise_routed_b200 as fm
import oracle
from gpu_helpers import ABS_TOL, REL_TOL, U32, EPS_EX2, EPS_RCP, _dec, _gamma, tok_rel

# Bound on the GPU's FP32 intermediate h (the derivation of the 128x128-block
# path's check, with the MX accumulation): g = sum over all K of exact
# products dec(a) 2^sa dec(w) 2^sw (powers of two: exact), summed by the
# tensor core in FP32 over the whole K, each addition taken as faithful
# (relative error < 2u): |g_gpu - g| <= gamma_K(2u) S_g, S_g the dot product
# of absolute values.  SiLU and the product with u as in that derivation.
# A GPU code is valid when its rounding interval at the GPU's own block
# scale meets [h - e_h, h + e_h] / 2^se_gpu; a GPU block scale is valid when
# it is the shared exponent of some maximum within max e_h of the oracle's.

def _mx_dequant(codes_u8, scale_bytes):
    """[n, K] codes with [n, K/32] UE8M0 bytes -> float64 values."""
    dec = torch.from_numpy(_dec())
    v = dec[torch.as_tensor(np.ascontiguousarray(codes_u8)).long()]
    sc = torch.pow(2.0, torch.as_tensor(np.ascontiguousarray(scale_bytes)).double() - 127.0)
    return v * sc.repeat_interleave(32, dim=-1)[..., : v.shape[-1]]


def _gpu_h_by_pair(g, wl, T):
    k, I, H = wl.k, wl.I, wl.H
    hc, hs = fm.moe_ffn_mx_intermediate(g["ws"], T, H, I, k)
    P = int(g["offsets"][-1].item())
    sp = g["sorted"][:P].cpu().numpy()
    gc = np.zeros((T * k, I), np.uint8)
    gs = np.zeros((T * k, I // 32), np.uint8)
    G = hs.shape[0]
    rows = hs.permute(1, 0, 2).reshape(T * k, G * 16)  # [P, chunk]
    gc[sp] = hc[:P, :I].cpu().numpy()
    gs[sp] = rows[:P, : I // 32].cpu().numpy()
    return gc.reshape(T, k, I), gs.reshape(T, k, I // 32)


def _mx_h_error_bound(wl, h, act_codes, act_scales, ids, toks):
    """e_h [n, k, I] bounding |h_gpu - h32| for the tokens ``toks``."""
    H, I = wl.H, wl.I
    cg = _gamma(H + 1, 2 * U32) * 1.0001
    A = _mx_dequant(np.asarray(act_codes)[toks], np.asarray(act_scales)[toks])
    Aabs = A.abs()
    n, k = ids.shape
    eh = np.zeros((n, k, I), np.float64)
    for e in np.unique(ids[ids >= 0]):
        ti, ji = np.nonzero(ids == e)
        a, aa = A[ti], Aabs[ti]
        Wg = _mx_dequant(h["w_gate"][e].numpy(), h["s_gate"][e].numpy())
        Wu = _mx_dequant(h["w_up"][e].numpy(), h["s_up"][e].numpy())
        gv, uv = (a @ Wg.T).numpy(), (a @ Wu.T).numpy()
        Eg, Eu = cg * (aa @ Wg.abs().T).numpy(), cg * (aa @ Wu.abs().T).numpy()
        sig = 1.0 / (1.0 + np.exp(-np.clip(gv, -700, 700)))
        silu = np.abs(gv * sig)
        eps_silu = 2 * U32 * (np.abs(gv) + Eg) + EPS_EX2 + EPS_RCP + 2 * U32
        au = np.abs(uv)
        eh[ti, ji] = (1.1 * Eg * au + silu * Eu + 1.1 * Eg * Eu
                      + (silu + 1.1 * Eg) * (au + Eu) * (eps_silu + U32) * 1.0001 + U32 * silu * au * 1.0001)
    return eh


def _shared_exp(amax):
    """The MX shared exponent of finite maxima (float64 array)."""
    with np.errstate(divide="ignore"):
        se = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8
    return np.where(amax > 0, np.clip(se, -127, 127), -127)


def check_mx_layer(wl, g, ref, h, toks):
    """GPU layer ``g`` against the oracle ``ref`` (want_h) on tokens toks."""
    T = g["out"].shape[0]
    ids = np.asarray(ref["ids"])[toks]
    w = np.asarray(ref["w"])[toks]
    gc, gs = _gpu_h_by_pair(g, wl, T)
    gc, gs = gc[toks], gs[toks]
    oc, osc, ohf = ref["h_codes"], ref["h_scales"], ref["h_fp32"].astype(np.float64)
    valid = ids >= 0
    I = wl.I
    eh = _mx_h_error_bound(wl, h, ref["codes"], ref["scales"], ids, toks)
    n, k = ids.shape
    # block scales
    amax_o = np.abs(ohf).reshape(n, k, I // 32, 32).max(-1)
    e_blk = eh.reshape(n, k, I // 32, 32).max(-1)
    lo = _shared_exp(np.maximum(amax_o - e_blk, 0.0)) + 127
    hi = _shared_exp(amax_o + e_blk) + 127
    gsv = gs.astype(np.int64)
    ok_s = (gsv >= lo) & (gsv <= hi)
    assert np.all(ok_s[valid]), f"{int((~ok_s[valid]).sum())} intermediate block scales outside the derived range"
    stats = {"scale_diffs": int(((gs != osc) & valid[..., None]).sum())}
    # codes: the rounding interval of the GPU code at the GPU scale must meet
    # the derived range of h / 2^se_gpu
    dec = _dec()
    vals = np.unique(dec[np.isfinite(dec)])
    vg = dec[gc]
    rank = np.searchsorted(vals, vg)
    below = np.where(rank > 0, (vals[np.maximum(rank - 1, 0)] + vg) / 2, -np.inf)
    above = np.where(rank < vals.size - 1, (vals[np.minimum(rank + 1, vals.size - 1)] + vg) / 2, np.inf)
    f = np.power(2.0, -(gsv - 127.0)).repeat(32, axis=-1)
    q_lo, q_hi = (ohf - eh) * f, (ohf + eh) * f
    ok_c = (below <= q_hi) & (above >= q_lo)
    ok_c |= ~valid[..., None]
    assert np.all(ok_c), f"{int((~ok_c).sum())} intermediate codes outside their derived rounding range"
    # output: literal tolerance widened by the effect of every differing
    # dequantised intermediate value
    v_g = _mx_dequant(gc, gs).numpy()
    v_o = _mx_dequant(oc, osc).numpy()
    diff = (v_g != v_o) & valid[..., None]
    stats["h_diffs"] = int(diff.sum())
    stats["h_values"] = int(valid.sum()) * I
    g_out = g["out"].double().cpu().numpy()[toks]
    r_out = np.asarray(ref["out"])
    allowance = np.zeros_like(g_out)
    pairs = np.nonzero(diff.any(-1))
    for e in np.unique(ids[pairs]) if diff.any() else []:
        Wd = np.abs(_mx_dequant(h["w_down"][e].numpy(), h["s_down"][e].numpy()).numpy())  # [H, I]
        for t, j in zip(*pairs):
            if ids[t, j] != e:
                continue
            dv = np.where(diff[t, j], np.abs(v_g[t, j] - v_o[t, j]), 0.0)
            allowance[t] += np.abs(wl.routed_scaling * w[t, j]) * (Wd @ dv)
    tol = REL_TOL * np.abs(r_out).max(axis=1, keepdims=True) + ABS_TOL
    err = np.abs(g_out - r_out)
    plain_bad = err > tol
    stats["plain_out_of_tol"] = int(plain_bad.sum())
    stats["worst_err_over_tol"] = float((err / tol).max()) if err.size else 0.0
    bad = err > tol + 1.001 * allowance
    assert not bad.any(), f"{int(bad.sum())} outputs outside tolerance + allowance; {stats}"
    assert np.all(allowance[plain_bad] > 0)
    stats["median_tok_rel"] = float(np.median(tok_rel(g_out, r_out))) if err.size else 0.0
    return stats


def _oracle_mx(wl, h, toks):
    return oracle.mx_moe_layer(h["x"], h["logits"], wl.k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"],
                               h["w_down"], h["s_down"], wl.routed_scaling, tokens=toks, want_h=True)


