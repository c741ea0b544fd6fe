"""GPU parity: routing ids, expert offsets and the permutation bit-exact
against the oracle; weights within 1e-6."""
import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle

pytestmark = pytest.mark.gpu


def gpu_route(logits, k):
    T, E = logits.shape
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    sp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_route(logits, k, ids, w, off, sp, ws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    return ids.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(), sp[: T * k].cpu().numpy()


def check(logits, k):
    ids, w, off, sp = gpu_route(logits, k)
    rid, rw = oracle.route(logits.cpu(), k)
    roff, rsp = oracle.permute(rid, logits.shape[1])
    assert np.array_equal(ids, rid)
    assert np.array_equal(off, roff)
    assert np.array_equal(sp, rsp)
    assert np.max(np.abs(w - rw), initial=0.0) <= 1e-6
    valid = rid >= 0
    if valid.any():
        np.testing.assert_allclose(w.sum(1)[valid.any(1)], 1.0, atol=1e-6)


@pytest.mark.parametrize("name", ["tiny", "small", "glm", "non128", "long"])
def test_route_workloads(name):
    wl = mi.WORKLOADS[name]
    check(mi.make_logits(wl, 0, "cuda"), wl.k)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (5, 3, 3), (129, 7, 2), (300, 64, 8), (1000, 1024, 32),
                                   (257, 300, 5), (4096 + 77, 160, 8)])
def test_route_shapes(T, E, k):
    g = torch.Generator(device="cuda").manual_seed(T * 31 + E)
    check(torch.randn((T, E), generator=g, device="cuda"), k)


def test_route_ties_and_masks():
    T, E, k = 300, 40, 6
    g = torch.Generator(device="cuda").manual_seed(3)
    lg = torch.randint(-3, 3, (T, E), generator=g, device="cuda").float()  # many ties
    lg[5] = float("-inf")
    lg[6, :] = float("-inf")
    lg[6, 11] = 2.0
    lg[7] = float("nan")
    lg[8, ::3] = float("nan")
    lg[9] = -0.0
    lg[9, ::2] = 0.0
    check(lg, k)


def test_route_top_k_zero_and_empty():
    ids, w, off, sp = gpu_route(torch.zeros((0, 16), device="cuda"), 4)
    assert np.all(off == 0)
    ids, w, off, sp = gpu_route(torch.randn((10, 16), device="cuda"), 0)
    assert np.all(off == 0)


def test_route_rejects_bad_args():
    lg = torch.zeros((4, 8), device="cuda")
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(fm.MoeError) as e:
        fm.moe_route(lg, 9, z, z, z, z, ws)  # top_k > E
    assert e.value.code == 1
    with pytest.raises(fm.MoeError) as e:
        fm.moe_route(lg, 2, z, z, z, z, ws[:8])  # workspace too small
    assert e.value.code == 4


def _route_quant(logits, x, k):
    T, E = logits.shape
    H = x.shape[1]
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    sp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    codes = torch.full((T, H), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((T, H // 128), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_route_quant(logits, x, k, ids, w, off, sp, codes, scales, ws)
    torch.cuda.synchronize()
    assert fm.moe_get_device_status(ws) == 0
    return ids, w, off, sp[: T * k], codes, scales


def _separate(logits, x, k):
    T, E = logits.shape
    H = x.shape[1]
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    sp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    codes = torch.full((T, H), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((T, H // 128), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_route(logits, k, ids, w, off, sp, ws)
    fm.moe_quant_act(x, codes, scales)
    torch.cuda.synchronize()
    return ids, w, off, sp[: T * k], codes, scales


@pytest.mark.parametrize("T,H,E,k", [(0, 256, 8, 2), (37, 256, 8, 0), (1, 128, 1, 1), (333, 640, 64, 8),
                                     (1000, 256, 1024, 32), (4096, 5120, 256, 8)])
def test_route_quant_equals_separate_calls(T, H, E, k):
    """The fused call (quantiser in the router's first launch) gives the
    separate calls' results bit for bit, including the degenerate T = 0 and
    top_k = 0 cases (top_k = 0 still quantises)."""
    g = torch.Generator(device="cuda").manual_seed(T * 7 + H + E + k)
    lg = torch.randn((T, E), generator=g, device="cuda")
    x = (torch.randn((T, H), generator=g, device="cuda") * 3).to(torch.bfloat16)
    if T > 10:
        x[3, 5] = float("nan")
        x[4] = 0
    a = _route_quant(lg, x, k)
    b = _separate(lg, x, k)
    for u, v, name in zip(a, b, ("ids", "w", "offsets", "sorted_pairs", "codes", "scales")):
        assert torch.equal(u.view(torch.int32) if u.dtype == torch.float32 else u,
                           v.view(torch.int32) if v.dtype == torch.float32 else v), name


def test_route_quant_codes_match_oracle():
    wl = mi.WORKLOADS["small"]
    lg = mi.make_logits(wl, 0, "cuda")
    x = mi.make_x(wl, 0, "cuda")
    ids, w, off, sp, codes, scales = _route_quant(lg, x, wl.k)
    rc, rs = oracle.quant_act(x.cpu())
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    rid, rw = oracle.route(lg.cpu(), wl.k)
    assert np.array_equal(ids.cpu().numpy(), rid)
