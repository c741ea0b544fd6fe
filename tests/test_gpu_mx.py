"""GPU parity of the MXFP8 variant with the oracle's MX rules (readings
M1-M3): the activation quantiser (moe_quant_act_mx) bit for bit, on the
workloads' activations and on special values (zeros, signed zeros, BF16
subnormals, the largest BF16 values, NaN and Inf); and the MX expert FFN
(moe_grouped_ffn_mx, then moe_combine) on whole layers, with the
intermediate's requantisation decisions checked against a bound derived from
the operands, as for the 128x128-block path."""
import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle
from gpu_helpers import ABS_TOL, REL_TOL, U32, EPS_EX2, EPS_RCP, _dec, _gamma, tok_rel

pytestmark = pytest.mark.gpu


def _gpu(x):
    T, H = x.shape
    codes = torch.full((T, H), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((T, H // 32), 0xAB, dtype=torch.uint8, device="cuda")
    fm.moe_quant_act_mx(x.cuda(), codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "small", "glm", "long"])
def test_mx_quant_matches_oracle(name):
    wl = mi.WORKLOADS[name]
    x = mi.make_x(wl, 0, "cuda", T=min(wl.T, 4096)).cpu()
    codes, scales = _gpu(x)
    rc, rs = oracle.mx_quant_act(x)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)


def test_mx_quant_special_values():
    T, H = 64, 256
    g = torch.Generator().manual_seed(3)
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    x[1, 5] = 0.0
    x[2, 32:64] = float("nan")
    x[3, 64:96] = float("inf")
    x[3, 100] = float("-inf")
    sub = torch.from_numpy(np.array([0x0001, 0x8003, 0x007F, 0x0040], np.uint16).view(np.int16)).view(torch.bfloat16)
    x[4, :4] = sub  # a block of BF16 subnormals (amax subnormal)
    x[4, 4:32] = 0.0
    x[5, :32] = torch.tensor(3.3895e38, dtype=torch.bfloat16)  # near the largest BF16
    x[5, 7] = -x[5, 7]
    x[6, :32] = torch.linspace(-448, 448, 32).to(torch.bfloat16)
    x[7, :32] = 1e-30
    codes, scales = _gpu(x)
    rc, rs = oracle.mx_quant_act(x)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)
    assert scales[2, 1] == 0xFF and np.all(codes[2, 32:64] == 0x7F)
    assert scales[0, 0] == 0 and codes[1, 0] == 0x80


def test_mx_quant_every_exponent():
    """A block maximum at every binade the BF16 range holds (normal and
    subnormal), with the other values spread below it."""
    rows = []
    g = torch.Generator().manual_seed(9)
    for e in range(-133, 128):
        r = torch.rand((32,), generator=g) * (2.0 ** e)
        r[0] = 2.0 ** e * 1.5 if e < 127 else 2.0 ** 127
        rows.append(r)
    x = torch.stack(rows).to(torch.bfloat16)
    x = torch.cat([x, x], dim=1)  # H = 64
    codes, scales = _gpu(x)
    rc, rs = oracle.mx_quant_act(x)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)


# ---------------------------------------------------------------------------
# MX expert FFN.
#
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


_packed: dict = {}


def packed(d):
    """The weight scales of d packed by moe_mx_pack_scales (once per tensor)."""
    key = tuple(d[n].data_ptr() for n in ("s_gate", "s_up", "s_down"))
    if key not in _packed:
        _packed.clear()
        _packed[key] = {n: fm.moe_mx_pack_scales(d[n]) for n in ("s_gate", "s_up", "s_down")}
    return _packed[key]


def test_mx_pack_scales():
    """The packed layout is a pure permutation of the checkpoint bytes (plus
    127 padding), on even and ragged K/32."""
    g = torch.Generator().manual_seed(5)
    for E, R, K in ((3, 70, 5120), (2, 33, 192), (1, 5, 32), (4, 192, 1536), (2, 8, 2080)):
        src = torch.randint(0, 255, (E, R, K // 32), generator=g, dtype=torch.uint8)
        dst = fm.moe_mx_pack_scales(src.cuda()).cpu().numpy()
        G = (K + 511) // 512
        want = np.full((E, R, G * 16), 127, np.uint8)
        want[:, :, : K // 32] = src.numpy()
        want = want.reshape(E, R, G, 16).transpose(0, 2, 1, 3)
        assert np.array_equal(dst, want)


def run_mx_layer(wl, d, rs=None):
    """Route (moe_route), quantise (moe_quant_act_mx), experts
    (moe_grouped_ffn_mx), combine (moe_combine) on CUDA tensors ``d``."""
    rs = wl.routed_scaling if rs is None else rs
    x, lg = d["x"], d["logits"]
    T, H = x.shape
    E, I, _ = d["w_gate"].shape
    k = wl.k
    dev = x.device
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    off = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    sp = torch.empty((max(T * k, 1),), dtype=torch.int32, device=dev)
    rws = torch.zeros((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device=dev)
    fm.moe_route(lg, k, ids, tw, off, sp, rws)
    codes = torch.empty((T, H), dtype=torch.uint8, device=dev)
    scales = torch.empty((T, H // 32), dtype=torch.uint8, device=dev)
    fm.moe_quant_act_mx(x, codes, scales)
    ws = torch.zeros((fm.moe_ffn_mx_workspace_bytes(T, H, I, E, k),), dtype=torch.uint8, device=dev)
    y = torch.zeros((T, k, H), dtype=torch.float32, device=dev)
    pk = packed(d)
    fm.moe_grouped_ffn_mx(codes, scales, ids, tw, off, sp, d["w_gate"], pk["s_gate"], d["w_up"], pk["s_up"],
                          d["w_down"], pk["s_down"], y, ws)
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    cws = torch.zeros((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device=dev)
    fm.moe_combine(y, ids, E, rs, out, None, cws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    assert fm.moe_get_device_status(cws) == 0
    return dict(ids=ids, w=tw, offsets=off, sorted=sp, codes=codes, scales=scales, ws=ws, y=y, out=out)


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


def _mx_case(name):
    wl = mi.WORKLOADS[name]
    d = mi.make_inputs_mx(wl, 0, "cuda")
    h = {key: v.cpu() for key, v in d.items()}
    return wl, d, h


@pytest.mark.parametrize("name", ["tiny", "small", "non128", "glm"])
def test_mx_layer_matches_oracle(name):
    wl, d, h = _mx_case(name)
    g = run_mx_layer(wl, d)
    T = wl.T
    ids_o, w_o = oracle.route(h["logits"], wl.k)
    assert np.array_equal(g["ids"].cpu().numpy(), ids_o)
    assert np.max(np.abs(g["w"].cpu().numpy() - w_o), initial=0.0) <= 1e-6
    off_o, sp_o = oracle.permute(ids_o, wl.E)
    assert np.array_equal(g["offsets"].cpu().numpy(), off_o)
    P = int(off_o[-1])
    assert np.array_equal(g["sorted"][:P].cpu().numpy(), sp_o[:P])
    if name in ("tiny", "small"):
        toks = np.arange(T)
    else:
        toks = np.sort(mi.sample_tokens(wl, torch.from_numpy(ids_o), n_random=48).numpy())
    ref = _oracle_mx(wl, h, toks)
    stats = check_mx_layer(wl, g, ref, h, toks)
    print(name, stats)
    # down projection + combine alone on the oracle's own intermediate: the
    # literal tolerance with no allowance
    k, I, H = wl.k, wl.I, wl.H
    Ip = (I + 127) // 128 * 128
    G = (Ip + 511) // 512
    SI = G * 16
    hc = np.zeros((T, k, Ip), np.uint8)
    hs = np.full((T, k, SI), 0xFF, np.uint8)  # bytes past I/32 must not be used
    hs[:, :, : I // 32] = 127
    hc[toks, :, :I] = ref["h_codes"]
    hs[toks, :, : I // 32] = ref["h_scales"]
    hc_s = np.zeros((T * k, Ip), np.uint8)
    hs_s = np.full((T * k, SI), 0xFF, np.uint8)
    hc_s[:P] = hc.reshape(T * k, Ip)[sp_o[:P]]
    hs_s[:P] = hs.reshape(T * k, SI)[sp_o[:P]]
    y = torch.zeros((T, k, H), dtype=torch.float32, device="cuda")
    cws = torch.zeros((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device="cuda")
    hs_g = np.ascontiguousarray(hs_s.reshape(T * k, G, 16).transpose(1, 0, 2))  # [G, P, 16]
    fm.moe_debug_grouped_down_mx(torch.from_numpy(hc_s).cuda(), torch.from_numpy(hs_g).cuda(), g["w"],
                                 g["offsets"], g["sorted"][: T * k], d["w_down"], packed(d)["s_down"], y, cws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(cws) == 0
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    fm.moe_combine(y, g["ids"], wl.E, wl.routed_scaling, out, None, cws)
    torch.cuda.synchronize()
    r = np.asarray(ref["out"])
    gd = out.double().cpu().numpy()[toks]
    tol = REL_TOL * np.abs(r).max(axis=1, keepdims=True) + ABS_TOL
    assert np.all(np.abs(gd - r) <= tol)


def test_mx_layer_row_invariance():
    """A row's output bits do not depend on the other rows of the call."""
    wl, d, h = _mx_case("small")
    g = run_mx_layer(wl, d)
    sub = {key: (v[:100] if key in ("x", "logits") else v) for key, v in d.items()}
    g2 = run_mx_layer(wl, sub)
    assert torch.equal(g2["out"], g["out"][:100])


def test_mx_layer_empty_and_masked():
    wl = mi.WORKLOADS["tiny"]
    d = mi.make_inputs_mx(wl, 2, "cuda")
    d["logits"][5] = float("-inf")
    g = run_mx_layer(wl, d)
    assert torch.all(g["out"][5] == 0)
    e = {key: (v[:0] if key in ("x", "logits") else v) for key, v in d.items()}
    g0 = run_mx_layer(wl, e)
    assert g0["out"].shape == (0, wl.H)
