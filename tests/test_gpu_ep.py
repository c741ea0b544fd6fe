"""Expert parallelism, emulated on one GPU: every virtual rank runs its own
kernels (plan, permutation, grouped FFN into its send rows) and the exchange
is done by slicing, exactly as the ranks would see it.  Each home rank's
rows must equal the single-GPU layer bit for bit (reading: slot rows summed
in slot order at home, so a row's bits do not depend on the sharding)."""
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
from fp8_blockwise_routed_b200 import ep

pytestmark = pytest.mark.gpu


def _single_gpu(wl, d):
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                         wl.routed_scaling, wl.T)
    out = layer.forward(d["x"], d["logits"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return out


def _shard(d, r, world, E):
    per = E // world
    return tuple(d[n][r * per:(r + 1) * per].contiguous()
                 for n in ("w_gate", "s_gate", "w_up", "s_up", "w_down", "s_down"))


def _emulate(wl, d, world):
    T, k = wl.T, wl.k
    ranks = [ep.ExpertParallelMoE(*_shard(d, r, world, wl.E), wl.E, k, wl.routed_scaling, T, rank=r, world=world)
             for r in range(world)]
    T_home = ep.home_tokens(T, world)
    sends, counts = [], []
    for m in ranks:  # each rank's side up to its send rows
        codes, scales, ids, tw = m.codes[:T], m.scales[:T], m.ids[:T], m.tw[:T]
        fm.moe_route_quant(d["logits"], d["x"], k, ids, tw, m.offsets, m.sorted[:T * k], codes, scales, m.ws_route)
        fm.moe_ep_plan(ids, wl.E, world, m.rank, T_home, m.local_ids[:T], m.send_rows[:T * k], m.recv_rows[:T_home],
                       m.offs_oh, m.offs_ho, m.ws_ep)
        fm.moe_permute(m.local_ids[:T], m.E_local, m.offsets_local, m.sorted_local[:T * k], m.ws_perm)
        fm.moe_grouped_ffn_rows(codes, scales, m.local_ids[:T], tw, m.offsets_local, m.sorted_local[:T * k], *m.w,
                                m.send[:T * k], m.send_rows[:T * k], m.ws_ffn)
        sends.append(m.send)
        counts.append(m.counts(T))
    outs = []
    for h, m in enumerate(ranks):  # the exchange as slicing, then the home sums
        parts = []
        for o in range(world):
            sc = counts[o][0]
            start = sum(sc[:h])
            parts.append(sends[o][start:start + sc[h]])
            assert sc[h] == counts[h][1][o]  # both sides agree on the row count
        recv = torch.cat(parts) if sum(p.shape[0] for p in parts) else torch.zeros((1, wl.H), device="cuda")
        t0, t1 = min(T, h * T_home), min(T, (h + 1) * T_home)
        out = torch.empty((t1 - t0, wl.H), dtype=torch.float32, device="cuda")
        fm.moe_combine_rows(recv.contiguous(), m.recv_rows[:t1 - t0], wl.routed_scaling, out, None, m.ws_comb)
        outs.append(out)
    torch.cuda.synchronize()
    for m in ranks:
        assert m.device_status() == 0
    return torch.cat(outs)


@pytest.mark.parametrize("name,world", [("small", 2), ("small", 4), ("non128", 4), ("glm", 8)])
def test_expert_parallel_equals_single_gpu(name, world):
    wl = mi.WORKLOADS[name]
    d = mi.make_inputs(wl, 0, "cuda")
    ref = _single_gpu(wl, d)
    got = _emulate(wl, d, world)
    assert torch.equal(got.view(torch.int32), ref.view(torch.int32))


def test_expert_parallel_ragged_homes_and_masked_tokens():
    """T not a multiple of world, tokens whose every logit is -inf (no slot)."""
    wl = mi.WORKLOADS["small"].with_(T=1003)
    d = mi.make_inputs(wl, 3, "cuda")
    d["logits"][7] = float("-inf")
    d["logits"][500, :] = float("-inf")
    d["logits"][500, 3] = 1.0  # a single selectable expert
    ref = _single_gpu(wl, d)
    got = _emulate(wl, d, 4)
    assert torch.equal(got.view(torch.int32), ref.view(torch.int32))
    assert torch.all(got[7] == 0)


def test_expert_parallel_world_one_class():
    wl = mi.WORKLOADS["tiny"]
    d = mi.make_inputs(wl, 0, "cuda")
    ref = _single_gpu(wl, d)
    m = ep.ExpertParallelMoE(*_shard(d, 0, 1, wl.E), wl.E, wl.k, wl.routed_scaling, wl.T)
    out = m.forward(d["x"], d["logits"])
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))


def test_ep_plan_rejects_bad_arguments():
    ids = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    ws = torch.empty((fm.moe_ep_plan_workspace_bytes(8, 2, 3),), dtype=torch.uint8, device="cuda")
    with pytest.raises(fm.MoeError):  # 8 experts do not split over 3 ranks
        fm.moe_ep_plan(ids, 8, 3, 0, 3, z, z, z, z, z, ws)
    with pytest.raises(fm.MoeError):  # homes do not cover the tokens
        fm.moe_ep_plan(ids, 9, 3, 0, 2, z, z, z, z, z, ws)


def test_expert_parallel_against_oracle():
    """Two emulated ranks on the tiny workload, compared with the oracle at the
    method's tolerance (the other tests compare with the single-GPU layer bit
    for bit); tokens the oracle routes nowhere are exact zeros."""
    import numpy as np

    import oracle
    from gpu_helpers import assert_close_rows

    wl = mi.WORKLOADS["tiny"]
    d = mi.make_inputs(wl, 0, "cuda")
    h = {k: v.cpu() for k, v in d.items()}
    ref = oracle.moe_layer(h["x"], h["logits"], wl.k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"], h["w_down"],
                           h["s_down"], wl.routed_scaling)
    got = _emulate(wl, d, 2)
    assert_close_rows(got, ref["out"])
    assert np.all(ref["out"][np.all(ref["ids"] < 0, axis=1)] == 0)
