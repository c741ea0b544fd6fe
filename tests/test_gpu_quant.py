"""GPU parity: E4M3 encoder and activation quantiser, bit-exact against the
oracle (codes and FP32 scales compared as bits)."""
import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle
from gpu_helpers import inputs

pytestmark = pytest.mark.gpu


def test_encoder_bits_sampled_all_patterns():
    """FP32 bit patterns spread over the whole 2^32 space (stride 251), plus
    every code value, their midpoints and the specials: hardware
    cvt.rn.satfinite against the oracle's nearest-value search."""
    pats = np.arange(0, 2**32, 251, dtype=np.uint64).astype(np.uint32)
    vals = oracle.e4m3_decode_all().astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    extra = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 448.0, 464.0, -464.0, 1e-45, -1e-45], np.float32)
    x = np.concatenate([pats.view(np.float32), vals, mids, extra])
    finite = ~np.isnan(x)
    x = x[finite]  # NaN payloads are covered by the quantiser's own rule
    xd = torch.from_numpy(x).cuda()
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    fm.moe_debug_encode(xd, out)
    got = out.cpu().numpy()
    want = oracle.e4m3_encode_array(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (x[bad[:8]], got[bad[:8]], want[bad[:8]])


def _quant(x):
    T, H = x.shape
    codes = torch.empty((T, H), dtype=torch.uint8, device="cuda")
    scales = torch.empty((T, H // 128), dtype=torch.float32, device="cuda")
    fm.moe_quant_act(x, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "small", "glm", "non128", "long"])
def test_quant_act_bit_exact(name):
    wl = mi.WORKLOADS[name]
    T = wl.T if name != "long" else 4096 + 37  # a 4096-row tile plus a ragged tail
    x = mi.make_x(wl, 0, "cuda", T=T)
    codes, scales = _quant(x)
    rc, rs = oracle.quant_act(x.cpu())
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))


def test_quant_act_special_values():
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn((19, 1024), generator=g, device="cuda")
    x[0, :128] = 0.0
    x[1, 5] = float("nan")
    x[2, 130] = float("inf")
    x[3, 300] = float("-inf")
    x[4, 512:640] = 1e-39                     # BF16 subnormals
    x[5, 640:768] = torch.linspace(-3e38, 3e38, 128)
    x[6] *= 1e-30
    x[7, ::2] = -0.0
    x[8, 0] = 448.0 * 2 ** -120
    xb = x.to(torch.bfloat16)
    codes, scales = _quant(xb)
    rc, rs = oracle.quant_act(xb.cpu())
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))


def test_quant_act_empty():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    codes, scales = _quant(x)
    assert codes.shape == (0, 256)


def test_quant_act_rejects_bad_width():
    x = torch.zeros((4, 200), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fm.MoeError) as e:
        fm.moe_quant_act(x, torch.empty((4, 200), dtype=torch.uint8, device="cuda"),
                         torch.empty((4, 2), dtype=torch.float32, device="cuda"))
    assert e.value.code == 1


def test_quant_act_every_amax_mantissa_across_binades():
    """Groups whose maximum is each of the 128 BF16 mantissas at amax
    exponents from the subnormals through the largest binade, including
    both sides of amax = 448 * 2^-100 (where the kernel switches between its
    divide-free quotient and the divide).  The other 127 values of a group are
    random BF16 patterns of magnitude <= amax spread over 40 binades below it,
    with signed zeros.  Codes and scales bit-exact against the oracle."""
    rng = np.random.default_rng(11)
    exps = [0, 1, 2, 30, 33, 34, 35, 36, 37, 38, 60, 100, 120, 126, 127, 128, 135, 200, 240, 253, 254]
    groups = []
    for e in exps:
        for m in range(128):
            if e == 0 and m == 0:
                continue
            amax = (e << 7) | m
            lo = max(0, e - 40)
            ex = rng.integers(lo, e + 1, size=127)
            mant = rng.integers(0, 128, size=127)
            top = ex == e
            mant[top] = rng.integers(0, m + 1, size=int(top.sum()))
            mag = (ex << 7) | mant
            mag[rng.random(127) < 0.03] = 0
            g = np.concatenate([[amax], mag]).astype(np.uint16)
            g |= (rng.random(128) < 0.5).astype(np.uint16) << 15
            rng.shuffle(g)
            groups.append(g)
    n = len(groups)
    per_row = 8
    n_rows = (n + per_row - 1) // per_row
    bits = np.zeros((n_rows * per_row, 128), np.uint16)
    bits[:n] = np.stack(groups)
    bits = bits.reshape(n_rows, per_row * 128)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales = _quant(x)
    rc, rs = oracle.quant_act(x.cpu())
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))
