"""Pins for the oracle's routing and permutation (CPU only).

Routing: top-k experts per token with normalised weights ("Exact AVX2 FP8
arithmetic conversion avoids costly LUT gathers", "Real-checkpoint
measurements": top-eight routes and normalised routing weights), softmax per
the tiny workload's statement.  Permutation: the stable grouping of (token,
slot) pairs by expert that the grouped gate/up call consumes ("GLM-5.3-Flash
EXL3 on CUDA: a whole prompt pass routes its experts in one call", commit
text: plan, grouped gate and up, grouped down, combine).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from dense_reference import route_full_sort


@pytest.mark.parametrize("name", ["tiny", "small", "non128", "glm"])
def test_route_vs_full_sort(name):
    wl = mi.WORKLOADS[name]
    T = min(wl.T, 512)
    lg = mi.make_logits(wl, 0, "cpu", T=T)
    ids, w = oracle.route(lg, wl.k)
    ids_ref, w_ref = route_full_sort(lg, wl.k)
    assert np.array_equal(ids, ids_ref)
    assert np.max(np.abs(w - w_ref)) < 1e-15
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-15)
    assert np.all(np.diff(w, axis=1) <= 0)  # weights descend with slot


def test_route_special_logits():
    E, k = 10, 4
    lg = torch.zeros((6, E))
    lg[0] = torch.tensor([1, 3, 3, 2, 3, 0, 0, 0, 0, 0.0])       # ties -> lower id first
    lg[1] = float("-inf")                                           # nothing selectable
    lg[2] = float("-inf"); lg[2, 7] = 5.0; lg[2, 2] = 1.0          # fewer than k selectable
    lg[3] = float("nan"); lg[3, 4] = -1.0                           # NaN never selected
    lg[4] = torch.arange(E, dtype=torch.float32)                    # strictly increasing
    lg[5, 3] = 1e30                                                 # dominant logit
    ids, w = oracle.route(lg, k)
    assert ids[0].tolist() == [1, 2, 4, 3]
    assert ids[1].tolist() == [-1, -1, -1, -1] and np.all(w[1] == 0)
    assert ids[2].tolist() == [7, 2, -1, -1]
    assert ids[3].tolist() == [4, -1, -1, -1] and w[3, 0] == 1.0
    assert ids[4].tolist() == [9, 8, 7, 6]
    assert ids[5, 0] == 3 and w[5, 0] == 1.0 and np.all(w[5, 1:] == 0.0)
    # softmax over the selected logits == full softmax renormalised
    e = np.exp(np.array([3, 3, 3, 2.0]) - 3)
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=0, atol=1e-16)


def test_route_top_k_equals_E():
    lg = torch.randn((5, 6), generator=torch.Generator().manual_seed(0))
    ids, w = oracle.route(lg, 6)
    for t in range(5):
        assert sorted(ids[t].tolist()) == list(range(6))
        full = torch.softmax(lg[t].double(), 0).numpy()
        np.testing.assert_allclose(w[t], full[ids[t]], atol=1e-15)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (64, 2, 8), (300, 8, 64), (1000, 8, 256)])
def test_permute_vs_stable_argsort(T, k, E):
    rng = np.random.default_rng(T)
    ids = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    off, sp = oracle.permute(ids, E)
    flat = ids.reshape(-1)
    valid = np.nonzero(flat >= 0)[0]
    order = valid[np.argsort(flat[valid], kind="stable")]
    P = valid.size
    assert off[-1] == P and off[0] == 0
    assert np.all(np.diff(off) >= 0)
    assert np.array_equal(sp[:P], order)
    assert np.all(sp[P:] == -1)
    counts = np.bincount(flat[valid], minlength=E)
    assert np.array_equal(np.diff(off), counts)
    # experts with no pairs have equal offsets
    assert np.all((np.diff(off) == 0) == (counts == 0))


def test_permute_all_empty():
    ids = np.full((7, 3), -1, np.int32)
    off, sp = oracle.permute(ids, 5)
    assert np.all(off == 0) and np.all(sp == -1)
