"""The combine fused into the down GEMM (moe_grouped_ffn_combine): the same
bits as moe_grouped_ffn followed by moe_combine, whatever the order in which
a token's slot rows arrive."""
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi

pytestmark = pytest.mark.gpu


def _prepare(wl, d):
    T, H, E, k = wl.T, wl.H, wl.E, wl.k
    codes = torch.empty((T, H), dtype=torch.uint8, device="cuda")
    scales = torch.empty((T, H // 128), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty((E + 1,), dtype=torch.int32, device="cuda")
    sp = torch.empty((T * k,), dtype=torch.int32, device="cuda")
    wsr = torch.empty((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_route_quant(d["logits"], d["x"], k, ids, w, off, sp, codes, scales, wsr)
    return codes, scales, ids, w, off, sp


def _w(d):
    return d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"]


def _both(wl, d, bf16=False):
    T, H, E, k = wl.T, wl.H, wl.E, wl.k
    codes, scales, ids, w, off, sp = _prepare(wl, d)
    ws = torch.empty((fm.moe_ffn_workspace_bytes(T, H, wl.I, E, k),), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, k, H), dtype=torch.float32, device="cuda")
    ref = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ref16 = torch.empty((T, H), dtype=torch.bfloat16, device="cuda") if bf16 else None
    wsc = torch.empty((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device="cuda")
    fm.moe_grouped_ffn(codes, scales, ids, w, off, sp, *_w(d), y, ws)
    fm.moe_combine(y, ids, E, wl.routed_scaling, ref, ref16, wsc)
    out = torch.full((T, H), 7.0, dtype=torch.float32, device="cuda")
    out16 = torch.empty((T, H), dtype=torch.bfloat16, device="cuda") if bf16 else None
    fm.moe_grouped_ffn_combine(codes, scales, ids, w, off, sp, *_w(d), y, wl.routed_scaling, out, out16, ws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    return ref, out, ref16, out16


@pytest.mark.parametrize("name", ["tiny", "small", "non128", "glm"])
def test_fused_combine_equals_separate_calls(name):
    wl = mi.WORKLOADS[name]
    d = mi.make_inputs(wl, 0, "cuda")
    ref, out, _, _ = _both(wl, d)
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))


def test_fused_combine_ragged_width_masked_tokens_bf16():
    """H = 640 (the last 256-column block has one half), tokens without any
    selectable expert (zero rows), routed_scaling 2.5, a BF16 copy."""
    wl = mi.WORKLOADS["small"].with_(H=640, T=777, routed_scaling=2.5)
    d = mi.make_inputs(wl, 1, "cuda")
    d["logits"][5] = float("-inf")
    d["logits"][600] = float("nan")
    ref, out, ref16, out16 = _both(wl, d, bf16=True)
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    assert torch.equal(out16.view(torch.int16), ref16.view(torch.int16))
    assert torch.all(out[5] == 0)


def test_fused_combine_deterministic_and_in_graph():
    wl = mi.WORKLOADS["small"]
    d = mi.make_inputs(wl, 2, "cuda")
    outs = [_both(wl, d)[1].clone() for _ in range(3)]
    assert all(torch.equal(o.view(torch.int32), outs[0].view(torch.int32)) for o in outs)
    plan = fm.LayerPlan(d["x"], d["logits"], wl.k, *_w(d), wl.routed_scaling, fused_combine=True)
    try:
        got = plan.launch()
        torch.cuda.synchronize()
        assert plan.device_status() == 0
        assert torch.equal(got.view(torch.int32), outs[0].view(torch.int32))
    finally:
        plan.close()


@pytest.mark.parametrize("name", ["tiny", "non128"])
def test_fused_combine_against_oracle(name):
    """The fused path against the oracle itself, at the method's tolerance on
    every element (these workloads meet the literal tolerance with no
    intermediate flips reaching it, so no allowance is needed)."""
    import oracle
    from gpu_helpers import assert_close_rows

    wl = mi.WORKLOADS[name]
    d = mi.make_inputs(wl, 0, "cuda")
    _, out, _, _ = _both(wl, d)
    h = {k: v.cpu() for k, v in d.items()}
    ref = oracle.moe_layer(h["x"], h["logits"], wl.k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"], h["w_down"],
                           h["s_down"], wl.routed_scaling)
    assert_close_rows(out, ref["out"])
