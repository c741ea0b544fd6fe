"""CPU tests of the MXFP8 layer check itself (mx_check.check_mx_layer): the
oracle's own intermediate, laid out as the CUDA workspace holds it, passes
with no differences, and planted GPU-side mistakes (a code moved far from
its value, a wrong block scale, a code moved across a boundary that is not
near, an output beyond the tolerance) are rejected.  The GPU's intermediate
accessor is replaced by one that returns these arrays; nothing here runs
CUDA."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mx_check
import oracle


def _case(name="tiny"):
    wl = mi.WORKLOADS[name] if name in mi.WORKLOADS else mi.Workload(name, 24, 256, 4, 2, 192, 1.5, "normal",
                                                                      "normal")
    d = mi.make_inputs_mx(wl, 0, "cpu")
    toks = np.arange(wl.T)
    ref = mx_check._oracle_mx(wl, d, toks)
    off, sp = oracle.permute(ref["ids"], wl.E)
    P = int(off[-1])
    T, k, I = wl.T, wl.k, wl.I
    Ip = (I + 127) // 128 * 128
    G = (Ip + 511) // 512
    codes = np.zeros((T * k, Ip), np.uint8)
    rows = np.full((T * k, G * 16), 0xFF, np.uint8)  # padding chunks must not matter
    codes[:P, :I] = ref["h_codes"].reshape(T * k, I)[sp[:P]]
    rows[:P, : I // 32] = ref["h_scales"].reshape(T * k, I // 32)[sp[:P]]
    g = {"ws": None, "offsets": torch.from_numpy(off), "sorted": torch.from_numpy(sp),
         "out": torch.from_numpy(ref["out"].copy())}
    return wl, d, ref, g, codes, rows, sp, P


def _check(monkeypatch, wl, d, ref, g, codes, rows):
    G = rows.shape[1] // 16
    scales = np.ascontiguousarray(rows.reshape(-1, G, 16).transpose(1, 0, 2))
    monkeypatch.setattr(mx_check.fm, "moe_ffn_mx_intermediate",
                        lambda ws, T, H, I, k: (torch.from_numpy(codes), torch.from_numpy(scales)))
    return mx_check.check_mx_layer(wl, g, ref, d, np.arange(wl.T))


@pytest.mark.parametrize("name", ["tiny", "i192"])
def test_oracle_intermediate_passes(monkeypatch, name):
    wl, d, ref, g, codes, rows, sp, P = _case(name)
    st = _check(monkeypatch, wl, d, ref, g, codes, rows)
    assert st["h_diffs"] == 0 and st["scale_diffs"] == 0 and st["plain_out_of_tol"] == 0


def _big_element(codes, P, I):
    """A row and column whose code has a large magnitude (far from zero)."""
    mag = codes[:P, :I] & 0x7F
    r, c = np.unravel_index(np.argmax(mag), mag.shape)
    return r, c


def test_far_code_is_rejected(monkeypatch):
    wl, d, ref, g, codes, rows, sp, P = _case()
    r, c = _big_element(codes, P, wl.I)
    codes[r, c] ^= 0x20  # exponent field changed: far from the value
    with pytest.raises(AssertionError, match="rounding range"):
        _check(monkeypatch, wl, d, ref, g, codes, rows)


def test_adjacent_code_far_from_boundary_is_rejected(monkeypatch):
    wl, d, ref, g, codes, rows, sp, P = _case()
    r, c = _big_element(codes, P, wl.I)
    codes[r, c] = (codes[r, c] & 0x80) | ((codes[r, c] & 0x7F) - 1)  # the next code down
    with pytest.raises(AssertionError, match="rounding range"):
        _check(monkeypatch, wl, d, ref, g, codes, rows)


def test_wrong_block_scale_is_rejected(monkeypatch):
    wl, d, ref, g, codes, rows, sp, P = _case()
    rows[3, 1] += 2
    with pytest.raises(AssertionError, match="block scales"):
        _check(monkeypatch, wl, d, ref, g, codes, rows)


def test_output_beyond_tolerance_is_rejected(monkeypatch):
    wl, d, ref, g, codes, rows, sp, P = _case()
    out = g["out"].numpy()
    t = int(np.argmax(np.abs(out).max(axis=1)))
    out[t, 7] += 3e-3 * np.abs(out[t]).max() + 2e-3
    with pytest.raises(AssertionError, match="outputs outside tolerance"):
        _check(monkeypatch, wl, d, ref, g, codes, rows)
