"""The whole layer behind one call (moe_layer) and captured in a CUDA graph
(moe_layer_plan): bit-identical to the three separate calls, replayable
with new inputs, and with stage events recorded inside the graph."""
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi

pytestmark = pytest.mark.gpu


def _inputs(name, seed=0):
    wl = mi.WORKLOADS[name]
    return wl, mi.make_inputs(wl, seed, "cuda")


def _three_calls(wl, d, out_bf16=None):
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                         wl.routed_scaling, wl.T)
    out = layer.forward(d["x"], d["logits"], out_bf16=out_bf16).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return out


def _w(d):
    return d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"]


@pytest.mark.parametrize("name", ["tiny", "small", "non128"])
def test_layer_call_equals_three_calls(name):
    wl, d = _inputs(name)
    ref = _three_calls(wl, d)
    out = torch.full_like(ref, 7.0)
    ws = torch.empty((fm.moe_layer_workspace_bytes(wl.T, wl.H, wl.I, wl.E, wl.k),), dtype=torch.uint8,
                     device="cuda")
    fm.moe_layer(d["logits"], d["x"], wl.k, *_w(d), wl.routed_scaling, out, None, ws)
    torch.cuda.synchronize()
    assert fm.moe_layer_get_device_status(ws, wl.T, wl.H, wl.I, wl.E, wl.k) == 0
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("name", ["small", "glm"])
def test_plan_equals_three_calls_and_replays(name):
    wl, d = _inputs(name)
    ref = _three_calls(wl, d)
    x = torch.empty_like(d["x"])
    lg = torch.empty_like(d["logits"])
    plan = fm.LayerPlan(x, lg, wl.k, *_w(d), wl.routed_scaling)
    try:
        # a first batch of other inputs, then the reference batch, through the
        # same graph: the replay reads whatever the input buffers hold
        x.copy_(mi.make_x(wl, 1, "cuda"))
        lg.copy_(mi.make_logits(wl, 1, "cuda"))
        first = plan.launch().clone()
        x.copy_(d["x"])
        lg.copy_(d["logits"])
        out = plan.launch()
        torch.cuda.synchronize()
        assert plan.device_status() == 0
        assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
        assert not torch.equal(first, out)
        again = plan.launch().clone()
        torch.cuda.synchronize()
        assert torch.equal(again.view(torch.int32), ref.view(torch.int32))  # deterministic replay
    finally:
        plan.close()


def test_plan_with_bf16_output_and_stage_events():
    wl, d = _inputs("small")
    ref_bf16 = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ref = _three_calls(wl, d, out_bf16=ref_bf16)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    out_bf16 = torch.empty_like(ref_bf16)
    plan = fm.LayerPlan(d["x"], d["logits"], wl.k, *_w(d), wl.routed_scaling, out_bf16=out_bf16,
                        stage_events=evs)
    try:
        out = plan.launch()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
        assert torch.equal(out_bf16.view(torch.int16), ref_bf16.view(torch.int16))
        spans = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
        assert all(s >= 0 for s in spans) and sum(spans) > 0
    finally:
        plan.close()


def test_plan_rejects_bad_arguments_without_capturing():
    wl, d = _inputs("tiny")
    x = d["x"][:, :200]  # H not a multiple of 128
    with pytest.raises(fm.MoeError):
        fm.LayerPlan(x.contiguous(), d["logits"], wl.k, *_w(d), 1.0)
    # the library stays usable: a valid plan on the same thread still works
    plan = fm.LayerPlan(d["x"], d["logits"], wl.k, *_w(d), 1.0)
    plan.launch()
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    plan.close()


@pytest.mark.parametrize("T,H,E,k,I", [
    (37, 640, 5, 1, 192),     # odd group count per token (5), T not a multiple of 8 tokens per block, k = 1
    (203, 1024, 12, 3, 320),  # k = 3, several 128-row tiles with ragged tails
    (1, 256, 4, 4, 128),      # one token, every expert taken
])
def test_layer_edge_shapes_equal_three_calls(T, H, E, k, I):
    """The layer's route writes the activation codes straight into the
    expert-ordered A rows (no gather): bit-identical to the separate calls
    on edge shapes, with fully masked tokens (every slot empty) and a NaN
    token among them."""
    wl = mi.Workload("edge", T, H, E, k, I, 1.5, "normal", "normal")
    d = mi.make_inputs(wl, 3, "cuda")
    if T > 2:
        d["logits"][1] = float("-inf")       # a token with no selectable expert
        d["logits"][T - 1, :] = float("-inf")
        d["x"][T // 2, 7] = float("nan")      # NaN stays in its token's row
    ref = _three_calls(wl, d)
    out = torch.full_like(ref, 7.0)
    ws = torch.empty((fm.moe_layer_workspace_bytes(T, H, I, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_layer(d["logits"], d["x"], k, *_w(d), wl.routed_scaling, out, None, ws)
    torch.cuda.synchronize()
    assert fm.moe_layer_get_device_status(ws, T, H, I, E, k) == 0
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    if T > 2:
        assert torch.all(out[1] == 0) and torch.all(out[T - 1] == 0)
        assert torch.isnan(out[T // 2]).all()
