"""Pins of the oracle's MXFP8 variant (readings M1-M3 in oracle/oracle.c):
UE8M0 decode over all 256 bytes against 2^(x-127); the 32-value block
quantiser against closed forms (power-of-two maxima, exactly representable
blocks, saturation, zeros, non-finite values) and against an independent
torch restatement; the MX layer against a dense brute-force evaluator that
decodes with torch's float8 type and evaluates every expert for every token."""
import math

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from dense_reference import decode_table, route_full_sort


def test_ue8m0_decode_exhaustive():
    for x in range(255):
        assert oracle.ue8m0_decode(x) == math.ldexp(1.0, x - 127)
    assert math.isnan(oracle.ue8m0_decode(255))
    assert oracle.ue8m0_decode(127) == 1.0 and oracle.ue8m0_decode(0) == 2.0 ** -127


@pytest.mark.parametrize("m", [-20, -9, -1, 0, 3, 8, 20])
def test_block_power_of_two_max(m):
    """amax = 2^m: shared exponent m - 8, so the maximum maps to 2^8 = 256,
    E4M3 code 0x78 (exponent field 15, mantissa 0)."""
    rng = np.random.default_rng(m + 40)
    x = (rng.uniform(-1, 1, 32) * 2.0 ** m).astype(np.float32)
    x[5] = np.float32(2.0 ** m)
    codes, sc = oracle.mx_quant_block(x)
    assert sc == m - 8 + 127
    assert codes[5] == 0x78


def test_block_exactly_representable():
    """A block whose values are E4M3 values times 2^se, with its maximum in
    [256, 448], round-trips: codes equal the representation, scale 2^se."""
    dec = decode_table().numpy()
    rng = np.random.default_rng(7)
    for se in (-10, -3, 0, 4):
        picks = rng.integers(0, 0x7F, 32)
        picks[0] = 0x7C  # 384 = 1.5 * 2^8: amax in [256, 512)
        sign = rng.integers(0, 2, 32) * 0x80
        codes_in = (picks | sign).astype(np.uint8)
        codes_in[0] = 0x7C
        x = (dec[codes_in] * 2.0 ** se).astype(np.float32)
        codes, sc = oracle.mx_quant_block(x)
        assert sc == se + 127
        vals = dec[codes] * 2.0 ** se
        assert np.array_equal(vals, x.astype(np.float64))


def test_block_saturates_above_448():
    """amax just below 2^(e+1): the scaled maximum is near 512 and saturates
    to 448 (0x7E), sign kept."""
    x = np.zeros(32, np.float32)
    x[0] = np.float32(1.99 * 2.0 ** 4)
    x[1] = -x[0]
    codes, sc = oracle.mx_quant_block(x)
    assert sc == 4 - 8 + 127
    assert codes[0] == 0x7E and codes[1] == 0xFE


def test_block_zero_and_nonfinite():
    z = np.zeros(32, np.float32)
    z[3] = -0.0
    codes, sc = oracle.mx_quant_block(z)
    assert sc == 0 and codes[3] == 0x80 and np.all(np.delete(codes, 3) == 0)
    for bad in (np.nan, np.inf, -np.inf):
        x = np.ones(32, np.float32)
        x[9] = bad
        codes, sc = oracle.mx_quant_block(x)
        assert sc == 0xFF and np.all(codes == 0x7F)


def _torch_mx_rows(v32: torch.Tensor):
    """Independent restatement with torch ops: rows [n, 32k] FP32 ->
    (codes, scale bytes, FP64 dequantised)."""
    n, C = v32.shape
    blk = v32.view(n, C // 32, 32)
    amax = blk.abs().amax(-1)
    _, ex = torch.frexp(amax)
    se = torch.where(amax == 0, torch.full_like(ex, -127), (ex - 9).clamp(-127, 127))
    q = (blk.double() * torch.pow(2.0, -se.double())[..., None]).clamp(-448, 448)
    codes = q.float().to(torch.float8_e4m3fn).view(torch.uint8).view(n, C)
    dq = decode_table()[codes.long()].view(n, C // 32, 32) * torch.pow(2.0, se.double())[..., None]
    return codes, (se + 127).to(torch.uint8), dq.view(n, C)


def test_block_vs_torch_restatement():
    rng = np.random.default_rng(11)
    rows = (rng.standard_normal((400, 32)) * np.exp(rng.uniform(-12, 12, (400, 1)))).astype(np.float32)
    t_codes, t_sc, _ = _torch_mx_rows(torch.from_numpy(rows))
    for i in range(rows.shape[0]):
        codes, sc = oracle.mx_quant_block(rows[i])
        assert sc == int(t_sc[i, 0])
        assert np.array_equal(codes, t_codes[i].numpy())


def test_quant_act_matches_blocks():
    wl = mi.WORKLOADS["tiny"]
    x = mi.make_x(wl, 0, "cpu")
    codes, scales = oracle.mx_quant_act(x)
    t_codes, t_sc, _ = _torch_mx_rows(x.float())
    assert np.array_equal(codes, t_codes.numpy()) and np.array_equal(scales, t_sc.numpy())


def _dense_mx(d, k, rs):
    """Every expert for every token, densely, from torch-decoded operands."""
    dec = decode_table()
    codes, sc, xd = _torch_mx_rows(d["x"].float())
    T, H = xd.shape
    E, I, _ = d["w_gate"].shape

    def deq(w, s):
        R, C = w.shape
        return dec[w.long()] * torch.pow(2.0, s.double() - 127).repeat_interleave(32, 1)[:, :C]

    ids, w = route_full_sort(d["logits"], k)
    out = torch.zeros((T, H), dtype=torch.float64)
    for e in range(E):
        G = xd @ deq(d["w_gate"][e], d["s_gate"][e]).T
        U = xd @ deq(d["w_up"][e], d["s_up"][e]).T
        h32 = (G / (1.0 + torch.exp(-G)) * U).to(torch.float32)
        _, _, hd = _torch_mx_rows(h32)
        O = hd @ deq(d["w_down"][e], d["s_down"][e]).T
        for t in range(T):
            for j in range(k):
                if ids[t, j] == e:
                    out[t] += w[t, j] * O[t]
    return rs * out.numpy(), ids


@pytest.mark.parametrize("name", ["tiny", "i192"])
def test_mx_layer_vs_dense_bruteforce(name):
    wl = mi.WORKLOADS["tiny"] if name == "tiny" else mi.Workload("i192", 24, 256, 4, 2, 192, 1.5, "normal",
                                                                    "normal")
    d = mi.make_inputs_mx(wl, 0, "cpu")
    ref = oracle.mx_moe_layer(d["x"], d["logits"], wl.k, d["w_gate"], d["s_gate"], d["w_up"], d["s_up"],
                              d["w_down"], d["s_down"], wl.routed_scaling)
    dense, ids = _dense_mx(d, wl.k, wl.routed_scaling)
    assert np.array_equal(ref["ids"], ids)
    err = np.abs(ref["out"] - dense)
    assert np.all(err <= 1e-12 * np.abs(dense).max(axis=1, keepdims=True) + 1e-300)


def test_mx_layer_invariants():
    wl = mi.WORKLOADS["tiny"]
    d = mi.make_inputs_mx(wl, 1, "cpu")
    lg = d["logits"].clone()
    lg[3] = float("-inf")
    args = (d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"])
    r1 = oracle.mx_moe_layer(d["x"], lg, wl.k, *args, 1.0)
    r2 = oracle.mx_moe_layer(d["x"], lg, wl.k, *args, 2.0)
    assert np.all(r1["out"][3] == 0)
    assert np.array_equal(r2["out"], 2 * r1["out"])
    # the MX and the 128x128-block layers are different quantisations of the
    # same FP32 weights: close, not equal
    b = mi.make_inputs(wl, 1, "cpu")
    rb = oracle.moe_layer(b["x"], lg, wl.k, b["w_gate"], b["s_gate"], b["w_up"], b["s_up"], b["w_down"],
                          b["s_down"], 1.0)
    rel = np.linalg.norm(rb["out"] - r1["out"]) / np.linalg.norm(rb["out"])
    assert 0 < rel < 0.1
