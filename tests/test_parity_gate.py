"""The GPU parity gate itself, exercised on the CPU: ``check_layer`` given the
oracle's own intermediate must pass, and given planted mistakes (a flipped
code far from its rounding boundary, a non-adjacent code, a 1 % scale error,
an output beyond the tolerance) must fail.  An adjacent flip whose exact
value lies within the derived bound of its boundary must be accepted.  The
"GPU" intermediate here is the oracle's, edited on the host: no CUDA code
runs, and the oracle is never fed anything but its own inputs."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
import moe_inputs as mi

WL = mi.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def case():
    h = mi.make_inputs(WL, 0, "cpu")
    ref = gh.oracle_layer(WL, h, want_h=True)
    return h, ref


def _run(monkeypatch, case, codes=None, scales=None, out=None):
    h, ref = case
    c = ref["h_codes"].copy() if codes is None else codes
    s = ref["h_scales"].copy() if scales is None else scales
    monkeypatch.setattr(gh, "gpu_intermediate_by_pair", lambda layer, T: (c, s))
    o = torch.from_numpy(ref["out"].copy() if out is None else out)
    return gh.check_layer(WL, None, o, ref, h)


def _far_element(ref):
    """A valid intermediate element whose oracle quotient sits near its code's
    value (far from both rounding boundaries), with a finite, non-extreme code."""
    q = ref["h_fp32"][..., : WL.I] / np.repeat(ref["h_scales"], 128, axis=-1)[..., : WL.I]
    dec = gh._dec()
    codes = ref["h_codes"][..., : WL.I]
    dist = np.abs(q - dec[codes])
    ok = (ref["ids"] >= 0)[..., None] & (np.abs(q) > 1) & (np.abs(q) < 400)
    dist = np.where(ok, dist, np.inf)
    return np.unravel_index(np.argmin(dist), dist.shape)


def test_own_intermediate_passes(monkeypatch, case):
    st = _run(monkeypatch, case)
    assert st["flips"] == 0 and st["plain_out_of_tol"] == 0


def test_adjacent_flip_far_from_boundary_fails(monkeypatch, case):
    _, ref = case
    t, j, c = _far_element(ref)
    codes = ref["h_codes"].copy()
    codes[t, j, c] += 1  # the next magnitude (|q| < 400: never the NaN code)
    with pytest.raises(AssertionError, match="derived distance"):
        _run(monkeypatch, case, codes=codes)


def test_non_adjacent_code_fails(monkeypatch, case):
    _, ref = case
    t, j, c = _far_element(ref)
    codes = ref["h_codes"].copy()
    codes[t, j, c] += 2
    with pytest.raises(AssertionError, match="not adjacent"):
        _run(monkeypatch, case, codes=codes)


def test_scale_error_fails(monkeypatch, case):
    _, ref = case
    scales = ref["h_scales"].copy()
    valid = np.nonzero(ref["ids"] >= 0)
    scales[valid[0][3], valid[1][3], 0] *= 1.01
    with pytest.raises(AssertionError, match="scale beyond"):
        _run(monkeypatch, case, scales=scales)


def test_output_beyond_tolerance_fails(monkeypatch, case):
    _, ref = case
    out = ref["out"].copy()
    out[5, 7] += 3e-3 * np.abs(out[5]).max() + 2e-3
    with pytest.raises(AssertionError, match="outside tolerance"):
        _run(monkeypatch, case, out=out)


def test_flip_within_derived_bound_is_accepted(monkeypatch, case):
    """The element whose oracle quotient lies closest (relative to its
    derived bound) to a rounding boundary, moved to the code across that
    boundary, with the output shifted by exactly the flip's effect."""
    h, ref = case
    dec = gh._dec()
    q = (ref["h_fp32"][..., : WL.I].astype(np.float32)
         / np.repeat(ref["h_scales"], 128, axis=-1)[..., : WL.I]).astype(np.float64)
    codes = ref["h_codes"][..., : WL.I]
    eh = gh.intermediate_error_bound(WL, h, ref["codes"], ref["scales"], ref["ids"], np.arange(WL.T))
    lim = eh / np.repeat(ref["h_scales"], 128, axis=-1)[..., : WL.I] + 4 * gh.U32 * np.abs(q)
    # neighbour across the nearer boundary: the next code in the direction of q
    up = np.where(q >= dec[codes], 1, -1) * np.where(codes & 0x80, -1, 1)
    nb = (codes.astype(np.int64) + up)
    okc = (nb & 0x7F) <= 0x7E
    nbc = np.clip(nb, 0, 255).astype(np.uint8)
    mid = (dec[codes] + dec[nbc]) / 2
    ratio = np.where((ref["ids"] >= 0)[..., None] & okc & ((codes & 0x7F) > 0), np.abs(q - mid) / lim, np.inf)
    t, j, c = np.unravel_index(np.argmin(ratio), ratio.shape)
    assert ratio[t, j, c] <= 1.0, "no element of this workload lies within its bound of a boundary"
    new = ref["h_codes"].copy()
    new[t, j, c] = nbc[t, j, c]
    e = ref["ids"][t, j]
    wd = h["w_down"].numpy()
    sd = h["s_down"].numpy()
    col = dec[wd[e, :, c]] * np.repeat(sd[e, :, c // 128].astype(np.float64), 128)[: WL.H]
    delta = (dec[nbc[t, j, c]] - dec[codes[t, j, c]]) * float(ref["h_scales"][t, j, c // 128])
    out = ref["out"].copy()
    out[t] += WL.routed_scaling * ref["w"][t, j] * delta * col
    st = _run(monkeypatch, case, codes=new, out=out)
    assert st["flips"] == 1 and st["max_flip_over_bound"] <= 1.0
