"""Pins for the oracle's E4M3 codec and group quantiser (CPU only).

Decode follows the page "Exact AVX2 FP8 arithmetic conversion avoids costly
LUT gathers", section "Semantics and scope" (exhaustive 256-encoding gate,
signed zeros, subnormals as mantissa * 2^-9, NaN to signed zero).  Encode and
the quantiser follow the readings stated in the oracle's header (round to
nearest even, saturating; scale = amax/448).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_page_rules.txt")


def _bits64(v: float) -> int:
    return int(np.array([v], np.float64).view(np.uint64)[0])


def test_decode_page_rules_golden():
    rows = 0
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            code, val, _rule = line.split()
            got = oracle.e4m3_decode(int(code, 16))
            want = float(val)
            assert _bits64(got) == _bits64(want), (code, got, want)  # sign of zero included
            rows += 1
    assert rows >= 20


def test_decode_exhaustive_vs_torch_float8():
    """All 256 encodings against torch's float8_e4m3fn -> float64 conversion
    (a library routine); the two NaN encodings must decode to signed zero."""
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        got = oracle.e4m3_decode(b)
        if b in (0x7F, 0xFF):
            assert math.isnan(ref[b])
            assert got == 0.0 and math.copysign(1.0, got) == (-1.0 if b & 0x80 else 1.0)
        else:
            assert _bits64(got) == _bits64(float(ref[b])), hex(b)


def test_decode_exhaustive_fp32_exact():
    """Every decoded value is exactly representable in FP32 (the page's claim
    for subnormals holds for all codes), and |value| <= 448."""
    vals = oracle.e4m3_decode_all()
    assert np.all(vals.astype(np.float32).astype(np.float64) == vals)
    assert np.max(np.abs(vals)) == 448.0
    # 126 distinct positive finite magnitudes + zero
    assert len(set(np.abs(vals).tolist())) == 127


def test_encode_roundtrip_all_codes():
    vals = oracle.e4m3_decode_all().astype(np.float32)
    codes = oracle.e4m3_encode_array(vals)
    for b in range(256):
        if b in (0x7F, 0xFF):
            continue
        assert codes[b] == b, hex(b)


def test_encode_vs_torch_dense_sweep():
    """A dense sweep of FP32 inputs against torch's float8 conversion (round
    to nearest even); torch does not saturate, so its input is clamped."""
    rng = np.random.default_rng(0)
    parts = [np.linspace(-460.0, 460.0, 2_000_001, dtype=np.float32),
             np.linspace(-0.05, 0.05, 500_001, dtype=np.float32),
             rng.standard_normal(500_000).astype(np.float32) * 30,
             (rng.integers(0, 2**32, 500_000, dtype=np.uint64).astype(np.uint32)).view(np.float32)]
    v = np.concatenate(parts)
    v = v[np.isfinite(v)]
    got = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(np.clip(v, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_encode_midpoints_ties_to_even():
    vals = np.sort(np.unique(np.abs(oracle.e4m3_decode_all())))
    n = 0
    for a, b in zip(vals[:-1], vals[1:]):
        mid = np.float32((a + b) / 2)  # exact: both have <= 4 significant bits
        assert float(mid) == (a + b) / 2
        ca, cb = oracle.e4m3_encode(a), oracle.e4m3_encode(b)
        want = ca if (ca & 1) == 0 else cb
        assert oracle.e4m3_encode(mid) == want
        assert oracle.e4m3_encode(-mid) == want | 0x80
        n += 1
    assert n == 126


def test_encode_special_values():
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(float("-inf")) == 0xFE
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E  # saturates instead of rounding to 480
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00  # below half the smallest subnormal
    assert oracle.e4m3_encode(-(2.0 ** -11)) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # tie between 0 and 2^-9 -> even
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02  # tie between 1 and 2 (x2^-9) -> even


# ---------------------------------------------------------------- quantiser


def test_quant_group_exact_representable():
    """A group of E4M3-representable values with amax 448 has scale exactly
    1 and codes equal to the values' own encodings."""
    rng = np.random.default_rng(1)
    vals = oracle.e4m3_decode_all()
    finite = vals[[b for b in range(256) if b not in (0x7F, 0xFF)]]
    x = rng.choice(finite, 128).astype(np.float32)
    x[17] = 448.0
    codes, s = oracle.quant_group(x)
    assert s == np.float32(1.0)
    for i in range(128):
        assert oracle.e4m3_decode(codes[i]) == float(x[i])


@pytest.mark.parametrize("m", [-20, -3, 1, 7])
def test_quant_group_power_of_two_scaling(m):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128).astype(np.float32)
    c0, s0 = oracle.quant_group(x)
    c1, s1 = oracle.quant_group((x * np.float32(2.0 ** m)).astype(np.float32))
    assert np.array_equal(c0, c1)
    assert s1 == np.float32(s0 * 2.0 ** m)


def test_quant_group_zero_and_nonfinite():
    c, s = oracle.quant_group(np.array([0.0, -0.0] * 64, np.float32))
    assert s == 1.0 and list(c[:2]) == [0x00, 0x80]
    x = np.ones(128, np.float32)
    x[5] = np.nan
    c, s = oracle.quant_group(x)
    assert math.isnan(s) and np.all(c == 0x7F)
    x[5] = np.inf
    c, s = oracle.quant_group(x)
    assert math.isnan(s) and np.all(c == 0x7F)


def test_quant_group_partial_and_tiny():
    # Partial group of 64 real columns; FP32 subnormal inputs (no flush to zero)
    x = np.full(64, 1e-42, np.float32)
    x[3] = -3e-42
    c, s = oracle.quant_group(x)
    assert s == np.float32(np.float32(3e-42) / np.float32(448.0)) and s != 0
    # Underflowing scale falls back to 1 and codes encode the raw values (0)
    x = np.full(16, 1.4e-45, np.float32)
    c, s = oracle.quant_group(x)
    assert s == 1.0 and np.all(c == 0)


def test_quant_act_vs_torch_ops():
    """Activation quantiser against the same rule written with torch ops
    (FP32 divide, float8 conversion), over BF16 inputs including outliers,
    subnormals and zeros."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn((37, 512), generator=g) * torch.exp(torch.randn((37, 1), generator=g) * 4)
    x[3, 10] = 0.0
    x[4, :128] = 0.0
    x[5, 128:256] = 1e-39  # BF16 subnormal range
    x[6, 300] *= 1e4
    xb = x.to(torch.bfloat16)
    codes, scales = oracle.quant_act(xb)
    xf = xb.float().view(37, 4, 128)
    amax = xf.abs().amax(dim=2)
    s = amax / torch.tensor(448.0)
    s = torch.where(s == 0, torch.ones_like(s), s)
    q = (xf / s[..., None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).reshape(37, 512)
    assert np.array_equal(scales, s.numpy())
    assert np.array_equal(codes, q.numpy())
