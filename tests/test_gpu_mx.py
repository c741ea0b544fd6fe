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
from gpu_helpers import ABS_TOL, REL_TOL
from mx_check import _oracle_mx, check_mx_layer

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
# MX expert FFN (the checks are in mx_check.py).

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


def test_routed_moe_mx_class_matches_calls():
    """RoutedMoEMX (scales packed at construction, four ABI calls per
    forward) gives the bits of the step-by-step calls, twice in a row."""
    wl, d, h = _mx_case("small")
    g = run_mx_layer(wl, d)
    layer = fm.RoutedMoEMX(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                           wl.routed_scaling, wl.T)
    for _ in range(2):
        out = layer.forward(d["x"], d["logits"])
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        assert torch.equal(out, g["out"])
