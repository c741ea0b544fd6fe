"""The shared-expert slot (the ninth slot of the pages' nine-slot plan):
routing and permutation bit-exact against the oracle, the routed kernels
never touch the shared slot's rows, and the layer output within tolerance of
the oracle with the shared row added after the routed scaling."""
import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle

pytestmark = pytest.mark.gpu


def _route_shared(lg, k):
    T, E = lg.shape
    ids = torch.full((T, k + 1), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k + 1), -7.0, dtype=torch.float32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    sp = torch.full((T * (k + 1),), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty((fm.moe_route_workspace_bytes(T, E, k + 1),), dtype=torch.uint8, device="cuda")
    fm.moe_route_shared(lg, k, ids, w, off, sp, ws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    return ids, w, off, sp


@pytest.mark.parametrize("name", ["tiny", "small", "glm"])
def test_route_shared_matches_oracle(name):
    wl = mi.WORKLOADS[name]
    lg = mi.make_logits(wl, 0, "cuda")
    ids, w, off, sp = _route_shared(lg, wl.k)
    rid, rw = oracle.route_shared(lg.cpu(), wl.k)
    roff, rsp = oracle.permute(rid, wl.E)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.max(np.abs(w.cpu().numpy() - rw)) <= 1e-6
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(sp.cpu().numpy(), rsp)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_layer_with_shared_slot(name):
    wl = mi.WORKLOADS[name].with_(routed_scaling=2.5)
    d = mi.make_inputs(wl, 2, "cuda")
    T, H, E, k = wl.T, wl.H, wl.E, wl.k
    codes = torch.empty((T, H), dtype=torch.uint8, device="cuda")
    scales = torch.empty((T, H // 128), dtype=torch.float32, device="cuda")
    fm.moe_quant_act(d["x"], codes, scales)
    ids, w, off, sp = _route_shared(d["logits"], k)
    g = torch.Generator(device="cuda").manual_seed(11)
    shared = torch.randn((T, H), generator=g, device="cuda")
    y = torch.zeros((T, k + 1, H), dtype=torch.float32, device="cuda")
    y[:, k, :] = shared  # the caller's shared-expert rows, written before the routed kernels run
    ws = torch.empty((fm.moe_ffn_workspace_bytes(T, H, wl.I, E, k + 1),), dtype=torch.uint8, device="cuda")
    fm.moe_grouped_ffn(codes, scales, ids, w, off, sp, d["w_gate"], d["s_gate"], d["w_up"], d["s_up"],
                       d["w_down"], d["s_down"], y, ws)
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    wsc = torch.empty((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device="cuda")
    fm.moe_combine_shared(y, ids, E, wl.routed_scaling, out, None, wsc)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0 and fm.moe_get_device_status(wsc) == 0
    # the shared slot's words are exactly as the caller wrote them
    assert torch.equal(y[:, k, :].view(torch.int32), shared.view(torch.int32))
    h = {n: v.cpu() for n, v in d.items()}
    ref = oracle.moe_layer_shared(h["x"], h["logits"], k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"],
                                  h["w_down"], h["s_down"], wl.routed_scaling, shared.cpu())["out"]
    got = out.double().cpu().numpy()
    tol = 2e-3 * np.abs(ref).max(axis=1, keepdims=True) + 1e-3
    assert np.all(np.abs(got - ref) <= tol)
    # with a zero shared row the output equals the layer without the slot
    y[:, k, :] = 0
    fm.moe_combine_shared(y, ids, E, wl.routed_scaling, out, None, wsc)
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], k,
                         wl.routed_scaling, T)
    plain = layer.forward(d["x"], d["logits"])
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
