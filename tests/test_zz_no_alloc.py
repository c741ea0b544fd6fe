"""moe_route_noalloc: the router for callers that cannot allocate device
memory (for example code running inside another runtime's execution hook,
which owns every device byte, or a path that cannot afford cudaMalloc's
implicit synchronisation).  It takes no workspace and uses the library's
static device scratch instead; its results must equal moe_route's.

This file is collected last on purpose: a failure here leaves every other
test already run.  It passes alone in a fresh process and after the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi

pytestmark = pytest.mark.gpu


def _outputs(T, E, k):
    return (torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -7.0, dtype=torch.float32, device="cuda"),
            torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
            torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda"))


def _with_workspace(logits, k):
    T, E = logits.shape
    ids, w, off, sp = _outputs(T, E, k)
    ws = torch.empty((fm.moe_route_workspace_bytes(T, E, k),), dtype=torch.uint8, device="cuda")
    fm.moe_route(logits, k, ids, w, off, sp, ws)
    return ids, w, off, sp


def _no_alloc(logits, k):
    """Through the C ABI directly: no workspace argument exists."""
    T, E = logits.shape
    ids, w, off, sp = _outputs(T, E, k)
    P = ctypes.c_void_p
    code = fm.lib().moe_route_noalloc(P(logits.data_ptr()), T, E, k, P(ids.data_ptr()), P(w.data_ptr()),
                                      P(off.data_ptr()), P(sp.data_ptr()),
                                      P(torch.cuda.current_stream().cuda_stream))
    assert code == 0, (code, fm.lib().moe_route_noalloc_error())
    return ids, w, off, sp


def test_noalloc_matches_route_on_two_calls_in_a_row():
    cases = [(mi.WORKLOADS["glm"], 0), (mi.WORKLOADS["small"], 1)]
    results = []
    for wl, seed in cases:  # two calls in a row, different shapes, same static scratch
        lg = mi.make_logits(wl, seed, "cuda")
        results.append((lg, wl.k, _no_alloc(lg, wl.k)))
    torch.cuda.synchronize()
    for lg, k, got in results:
        ref = _with_workspace(lg, k)
        torch.cuda.synchronize()
        T = lg.shape[0]
        # both run the same kernels: every output equal bit for bit
        for a, b, name in zip(got[:3], ref[:3], ("topk_ids", "topk_w", "expert_offsets")):
            assert torch.equal(a, b), name
        assert torch.equal(got[3][: T * k], ref[3][: T * k]), "sorted_pairs"
        assert np.all(np.diff(got[2].cpu().numpy()) >= 0)


def _scratch_need(T, E, k):
    """Scratch bytes of a call, by the formula the header states: 256 +
    ceil(T/128)*E*4 + T*top_k*4, each region 256-byte aligned."""
    a = lambda v: (v + 255) // 256 * 256  # noqa: E731
    nb = (max(T, 1) + 127) // 128
    return a(a(256 + nb * E * 4) + max(T, 1) * max(k, 1) * 4)


CAP = (1 << 20) + 4096  # the static array's size, as the header states


def test_noalloc_largest_documented_case():
    """T = 16384, E = 1024, top_k = 8: the case the header says fits."""
    T, E, k = 16384, 1024, 8
    assert _scratch_need(T, E, k) <= CAP
    g = torch.Generator(device="cuda").manual_seed(5)
    lg = torch.randn((T, E), device="cuda", generator=g)
    got = _no_alloc(lg, k)
    ref = _with_workspace(lg, k)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    E, k = 1024, 8
    T = next(t for t in range(16384, 40000, 128) if _scratch_need(t, E, k) > CAP)
    # the first 128-token step that no longer fits is rejected ...
    lg = torch.zeros((T, E), device="cuda")
    with pytest.raises(fm.MoeError) as e:
        fm.moe_route_noalloc(lg, k, *_outputs(T, E, k))
    assert e.value.code == 4
    assert "static array" in str(e.value)
    # ... and the size just below it still runs
    T0 = T - 128
    assert _scratch_need(T0, E, k) <= CAP
    lg0 = torch.zeros((T0, E), device="cuda")
    _no_alloc(lg0, k)
    torch.cuda.synchronize()


def test_noalloc_empty_inputs():
    """T = 0 and top_k = 0 route nothing; expert_offsets is written as zeros."""
    for T, k in ((0, 8), (50, 0)):
        lg = torch.randn((T, 64), device="cuda")
        _, _, off, _ = _no_alloc(lg, k)
        torch.cuda.synchronize()
        assert torch.equal(off, torch.zeros_like(off))
