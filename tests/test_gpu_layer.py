"""GPU parity of the whole layer (route -> quantise -> grouped FFN ->
combine) against the oracle, at sizes the oracle finishes in seconds (every
output element) and at the full workload sizes (sampled tokens); row
invariance, determinism, NaN isolation, degenerate cases and device-side
fault reporting."""
import numpy as np
import pytest
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
from gpu_helpers import (assert_close_rows, check_down_on_oracle_intermediate, check_layer, inputs, oracle_layer,
                         oracle_layer_h, run_layer, sha, tok_rel)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": mi.WORKLOADS["tiny"],
    # intermediate 192 zero-padded to 256, odd T
    "i192": mi.Workload("i192", 40, 384, 5, 3, 192, 1.5, "normal", "normal"),
    # several 128-row tiles per expert with ragged tails; three N tiles
    "tiles": mi.Workload("tiles", 700, 512, 4, 2, 384, 1.0, "normal_outliers", "normal"),
    # hidden not a multiple of 256 (half-empty last down tile), I=320
    "h640": mi.Workload("h640", 333, 640, 12, 4, 320, 0.5, "normal", "uniform"),
    # one expert, top-1: a dense FFN
    "dense": mi.Workload("dense", 150, 256, 1, 1, 256, 1.0, "normal", "normal"),
    # the largest hidden and intermediate widths the ABI accepts (H 16384,
    # I 8192: 128 K blocks for gate/up, 64 for down, 64 N tiles each)
    "maxdims": mi.Workload("maxdims", 16, 16384, 3, 2, 8192, 1.0, "normal", "normal"),
    # the most experts and slots the ABI accepts (E 1024, top-32): ~2 rows
    # per expert, one partly filled tile each, 32 slot rows per token
    "maxexperts": mi.Workload("maxexperts", 64, 256, 1024, 32, 128, 1.0, "normal", "normal"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small_every_element(name):
    wl = SMALL[name]
    d, h = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    assert layer.device_status() == 0
    ref = oracle_layer_h(wl, h)
    assert np.array_equal(layer.ids[: wl.T].cpu().numpy(), ref["ids"])
    assert np.array_equal(layer.codes[: wl.T].cpu().numpy(), ref["codes"])
    st = check_layer(wl, layer, out, ref, h)
    print(name, st)
    assert st["flip_rate"] < 1e-3
    assert st["median_tok_rel"] < 2e-2


@pytest.mark.parametrize("name", ["small", "non128"])
def test_layer_workload_every_element(name):
    wl = mi.WORKLOADS[name]
    d, h = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    assert layer.device_status() == 0
    ref = oracle_layer_h(wl, h)
    st = check_layer(wl, layer, out, ref, h)
    print(name, st)
    assert st["flip_rate"] < 1e-3


def _sampled(wl, layer):
    return mi.sample_tokens(wl, layer.ids[: wl.T].cpu()).numpy()


@pytest.mark.parametrize("name", ["glm", "long"])
def test_layer_workload_sampled(name):
    """Full-size call; the oracle evaluates a deterministic token sample (all
    outlier tokens, 256 seeded tokens, tokens of the most and least loaded
    experts)."""
    wl = mi.WORKLOADS[name]
    d, h = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    assert layer.device_status() == 0
    ids = layer.ids[: wl.T].cpu()
    toks = _sampled(wl, layer)
    ref = oracle_layer_h(wl, h, tokens=toks)
    assert np.array_equal(ids.numpy(), ref["ids"])
    st = check_layer(wl, layer, out, dict(ref, ids=ref["ids"][toks], w=ref["w"][toks]), h, tokens=toks)
    print(name, len(toks), st)
    assert st["flip_rate"] < 1e-3


@pytest.mark.parametrize("name", list(SMALL) + ["small", "non128", "glm", "long"])
def test_down_and_combine_on_oracle_intermediate(name):
    """Diagnostic of the down GEMM and the combine alone: the oracle's own
    intermediate codes and scales go into the CUDA down GEMM (a test hook)
    and the CUDA combine, so no requantisation decision can differ; every
    compared output must meet the method's literal tolerance
    |err| <= 2e-3 * ||row||_inf + 1e-3 with no allowance.  Full-size
    workloads compare the oracle's token sample."""
    wl = SMALL.get(name) or mi.WORKLOADS[name]
    d, h = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    assert layer.device_status() == 0
    toks = _sampled(wl, layer) if name in ("glm", "long") else None
    ref = oracle_layer_h(wl, h, tokens=toks)
    assert np.array_equal(layer.ids[: wl.T].cpu().numpy(), ref["ids"])
    st = check_down_on_oracle_intermediate(wl, layer, ref, h, tokens=toks)
    print(name, st)


@pytest.mark.parametrize("name", ["tiny", "tiles", "h640"])
def test_row_invariance(name):
    """A row's output bits do not depend on how many rows share the call:
    one call, calls over chunks of rows, and single rows."""
    wl = SMALL[name]
    d, _ = inputs(wl)
    _, full, _ = run_layer(wl, d)
    full = full.clone()
    chunk = 37
    parts = []
    for t0 in range(0, wl.T, chunk):
        dd = dict(d, x=d["x"][t0:t0 + chunk].contiguous(), logits=d["logits"][t0:t0 + chunk].contiguous())
        parts.append(run_layer(wl, dd)[1].clone())
    assert torch.equal(torch.cat(parts), full)
    for t in sorted({0, 1, wl.T // 2, wl.T - 1}):
        dd = dict(d, x=d["x"][t:t + 1].contiguous(), logits=d["logits"][t:t + 1].contiguous())
        assert torch.equal(run_layer(wl, dd)[1][0], full[t])


@pytest.mark.parametrize("name", ["glm", "non128", "long"])
def test_row_invariance_full_widths(name):
    """Row invariance at the full workloads' widths (GEMM tiling, zero-padded
    intermediate, K-block counts of the real shapes): sampled rows run alone
    give the bits of the same rows in the full call (the first, middle and
    last token, outlier tokens, a token of the least-loaded expert); the long
    prefill also as four 4,096-row calls against the one 16,384-row call."""
    wl = mi.WORKLOADS[name]
    d, _ = inputs(wl)
    layer, full, _ = run_layer(wl, d)
    full = full.clone()
    ids = layer.ids[: wl.T].cpu().numpy()
    del layer
    rows = {0, wl.T // 2, wl.T - 1}
    if wl.x_dist == "normal_outliers":
        rows |= set(mi.outlier_tokens(wl, 0).tolist()[:2])
    counts = np.bincount(ids[ids >= 0].ravel(), minlength=wl.E)
    active = np.nonzero(counts)[0]
    least = active[np.argmin(counts[active])]
    rows.add(int(np.nonzero((ids == least).any(axis=1))[0][0]))
    for t in sorted(rows):
        dd = dict(d, x=d["x"][t:t + 1].contiguous(), logits=d["logits"][t:t + 1].contiguous())
        assert torch.equal(run_layer(wl, dd)[1][0], full[t]), f"row {t}"
    if wl.T > 4096:
        for t0 in range(0, wl.T, 4096):
            dd = dict(d, x=d["x"][t0:t0 + 4096].contiguous(), logits=d["logits"][t0:t0 + 4096].contiguous())
            assert torch.equal(run_layer(wl, dd)[1], full[t0:t0 + 4096]), f"rows {t0}..{t0 + 4095}"


def test_row_invariance_4096_tiles():
    """The long-prefill statement: rows give the same bits whether a pass of
    8,192 rows runs as one call or as two 4,096-row calls."""
    wl = mi.WORKLOADS["small"].with_(T=8192)
    d, _ = inputs(wl, seed=1)
    _, full, _ = run_layer(wl, d)
    full = full.clone()
    for t0 in (0, 4096):
        dd = dict(d, x=d["x"][t0:t0 + 4096].contiguous(), logits=d["logits"][t0:t0 + 4096].contiguous())
        assert torch.equal(run_layer(wl, dd)[1], full[t0:t0 + 4096])


def test_determinism_hashes():
    wl = SMALL["tiles"]
    d, _ = inputs(wl)
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"],
                         wl.k, wl.routed_scaling, wl.T)
    hashes = set()
    for _ in range(5):
        out = layer.forward(d["x"], d["logits"])
        torch.cuda.synchronize()
        hashes.add((sha(out), sha(layer.ids[: wl.T]), sha(layer.sorted[: wl.T * wl.k])))
    assert len(hashes) == 1


def test_nan_stays_in_its_row():
    wl = SMALL["tiles"]
    d, _ = inputs(wl)
    _, base, _ = run_layer(wl, d)
    base = base.clone()
    x = d["x"].clone()
    x[17, 3] = float("nan")
    _, out, _ = run_layer(wl, dict(d, x=x))
    assert torch.isnan(out[17]).all()
    keep = torch.ones(wl.T, dtype=torch.bool, device="cuda")
    keep[17] = False
    assert torch.equal(out[keep], base[keep])


def test_degenerate_cases():
    wl = SMALL["i192"]
    d, h = inputs(wl)
    lg = d["logits"].clone()
    lg[4] = float("-inf")  # routed to no expert
    dd = dict(d, logits=lg)
    _, o1, b1 = run_layer(wl, dd, routed_scaling=1.0, bf16=True)
    o1 = o1.clone()
    _, o2, _ = run_layer(wl, dd, routed_scaling=2.0)
    assert torch.all(o1[4] == 0)
    assert torch.equal(o2, 2 * o1)
    assert torch.equal(b1, o1.to(torch.bfloat16))
    # T = 0
    d0 = dict(d, x=d["x"][:0], logits=d["logits"][:0])
    _, o0, _ = run_layer(wl, d0)
    assert o0.shape == (0, wl.H)


def test_experts_without_tokens():
    """Experts that receive no pairs (the non-128 workload masks 20%) and
    experts whose only tile is mostly padding."""
    wl = mi.WORKLOADS["non128"].with_(T=200)
    d, h = inputs(wl, seed=3)
    layer, out, _ = run_layer(wl, d)
    off = layer.offsets.cpu().numpy()
    masked = mi.masked_experts(wl, 3).numpy()
    assert np.all(np.diff(off)[masked] == 0)
    ref = oracle_layer(wl, h, want_h=True)
    check_layer(wl, layer, out, ref, h)


def test_device_status_bad_ids():
    wl = SMALL["tiny"]
    d, _ = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    ids = layer.ids[: wl.T].clone()
    ids[3, 0] = wl.E + 5
    ws = torch.empty((fm.moe_combine_workspace_bytes(),), dtype=torch.uint8, device="cuda")
    o = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    fm.moe_combine(layer.y[: wl.T], ids, wl.E, 1.0, o, None, ws)
    assert fm.moe_get_device_status(ws) & fm.DEV_BAD_EXPERT_ID


def test_device_status_bad_offsets():
    wl = SMALL["tiny"]
    d, _ = inputs(wl)
    layer, out, _ = run_layer(wl, d)
    off = layer.offsets.clone()
    off[2] = off[3] + 5  # not monotone
    y = torch.zeros_like(layer.y[: wl.T])
    fm.moe_grouped_ffn(layer.codes[: wl.T], layer.scales[: wl.T], layer.ids[: wl.T], layer.tw[: wl.T], off,
                       layer.sorted[: wl.T * wl.k], *layer.w, y, layer.ws_ffn)
    st = fm.moe_get_device_status(layer.ws_ffn)
    assert st & fm.DEV_BAD_OFFSETS
    assert not (st & fm.DEV_WAIT_TIMEOUT)
    assert torch.all(y == 0)


def test_exact_integer_layer():
    """Exact-arithmetic case: every value on the path is an integer the
    formats hold exactly, so the GPU output must equal an integer matmul bit
    for bit.  x rows hold 448 (column 0: activation scale exactly 1), 32 and 1
    (columns 1, 2); weight scales are 1; gate weights give g = 32 for every
    intermediate column, where SiLU(g) = g in FP32 (e^-32 is below half an
    ulp of 1); up weights give u = n mod 15, so h = 32 u is a multiple of 32
    up to 448 (E4M3-exact, and every 128-group's amax is 448: intermediate
    scale exactly 1); down weights are small integers; each token is routed
    to one expert (weight 1) and routed_scaling is 1."""
    T, H, I, E, k = 300, 256, 256, 4, 1
    dev = "cuda"
    x = torch.zeros((T, H), dtype=torch.float32)
    x[:, 0], x[:, 1], x[:, 2] = 448.0, 32.0, 1.0
    wg = torch.zeros((E, I, H))
    wg[:, :, 1] = 1.0                      # g_n = 32
    wu = torch.zeros((E, I, H))
    wu[:, :, 2] = (torch.arange(I) % 15).float()   # u_n = n mod 15
    g = torch.Generator().manual_seed(4)
    wd = torch.randint(-3, 4, (E, H, I), generator=g).float()
    logits = torch.full((T, E), -5.0)
    owner = torch.arange(T) % E
    logits[torch.arange(T), owner] = 5.0

    def codes(w):
        return w.to(torch.float8_e4m3fn).view(torch.uint8).to(dev)

    ones_gu = torch.ones((E, I // 128, H // 128), device=dev)
    ones_d = torch.ones((E, H // 128, I // 128), device=dev)
    layer = fm.RoutedMoE(codes(wg), ones_gu, codes(wu), ones_gu.clone(), codes(wd), ones_d, k, 1.0, T)
    out = layer.forward(x.to(torch.bfloat16).to(dev), logits.to(dev))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    h = (32 * (torch.arange(I) % 15)).to(torch.int64)                 # [I]
    want = torch.stack([wd[owner[t]].to(torch.int64) @ h for t in range(T)])  # [T, H]
    assert torch.equal(out.cpu(), want.to(torch.float32))
