"""Pins of the oracle's shared-expert slot (the ninth slot of the pages'
nine-slot plan): the routed part is unchanged, the extra slot is (E, 1), and
the shared row is added after the routed scaling."""
import numpy as np
import torch

import moe_inputs as mi
import oracle


def _w(d):
    return [d[k] for k in ("w_gate", "s_gate", "w_up", "s_up", "w_down", "s_down")]


def test_route_shared_appends_the_shared_slot():
    wl = mi.WORKLOADS["tiny"]
    lg = mi.make_logits(wl, 0, "cpu")
    ids, w = oracle.route(lg, wl.k)
    ids2, w2 = oracle.route_shared(lg, wl.k)
    assert ids2.shape == (wl.T, wl.k + 1)
    assert np.array_equal(ids2[:, :wl.k], ids) and np.all(ids2[:, wl.k] == wl.E)
    assert np.array_equal(w2[:, :wl.k], w) and np.all(w2[:, wl.k] == 1.0)
    # the shared id is outside the routed experts, so the permutation skips it
    off, sp = oracle.permute(ids2, wl.E)
    off0, _ = oracle.permute(ids, wl.E)
    assert off[-1] == off0[-1] == int((ids >= 0).sum())


def test_shared_rows_added_after_routed_scaling():
    wl = mi.WORKLOADS["tiny"].with_(routed_scaling=2.5)
    d = mi.make_inputs(wl, 1, "cpu")
    g = torch.Generator().manual_seed(5)
    shared = torch.randn((wl.T, wl.H), generator=g, dtype=torch.float32)
    res = oracle.moe_layer(d["x"], d["logits"], wl.k, *_w(d), wl.routed_scaling, want_slots=True)
    want = wl.routed_scaling * res["slots"].sum(axis=1) + shared.double().numpy()
    got = oracle.moe_layer_shared(d["x"], d["logits"], wl.k, *_w(d), wl.routed_scaling, shared)["out"]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    # a zero shared row leaves the routed layer's output exactly
    zero = oracle.moe_layer_shared(d["x"], d["logits"], wl.k, *_w(d), wl.routed_scaling,
                                   torch.zeros_like(shared))["out"]
    assert np.array_equal(zero, res["out"])
    # the scaling does not reach the shared row: scaling the routed part by 0
    # leaves exactly the shared rows
    only = oracle.moe_layer_shared(d["x"], d["logits"], wl.k, *_w(d), 0.0, shared)["out"]
    assert np.array_equal(only, shared.double().numpy())
