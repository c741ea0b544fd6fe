"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI binding and the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import hashlib

import numpy as np
import torch

import fp8_blockwise_routed_b200 as fm
import moe_inputs as mi
import oracle

# Output tolerance of the method's statement: |err| <= 2e-3 * ||row||_inf + 1e-3.
REL_TOL = 2e-3
ABS_TOL = 1e-3

_cache: dict = {}


def inputs(wl: mi.Workload, seed: int = 0, T: int | None = None):
    """CUDA tensors of a workload and CPU copies of the same bytes."""
    key = (wl, seed, T)
    if key not in _cache:
        if len(_cache) > 2:
            _cache.clear()
            torch.cuda.empty_cache()
        d = mi.make_inputs(wl, seed, "cuda", T=T)
        h = {k: v.cpu() for k, v in d.items()}
        _cache[key] = (d, h)
    return _cache[key]


def run_layer(wl: mi.Workload, d: dict, routed_scaling: float | None = None, bf16: bool = False):
    rs = wl.routed_scaling if routed_scaling is None else routed_scaling
    T = d["x"].shape[0]
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"],
                         wl.k, rs, max_tokens=max(T, 1))
    ob = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda") if bf16 else None
    out = layer.forward(d["x"], d["logits"], out_bf16=ob)
    torch.cuda.synchronize()
    return layer, out, ob


def assert_close_rows(gpu_out, ref_out, rows=None):
    g = gpu_out.detach().double().cpu().numpy() if hasattr(gpu_out, "detach") else np.asarray(gpu_out)
    if rows is not None:
        g = g[rows]
    ref = np.asarray(ref_out)
    tol = REL_TOL * np.abs(ref).max(axis=1, keepdims=True) + ABS_TOL
    err = np.abs(g - ref)
    bad = err > tol
    assert not bad.any(), (
        f"{int(bad.sum())} of {bad.size} outputs out of tolerance; worst err {err.max():.3e}, "
        f"worst err/tol {(err / tol).max():.3f}")
    return err, tol


def tok_rel(gpu_out, ref_out):
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    return np.linalg.norm(g - r, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-300)


def sha(t: torch.Tensor) -> str:
    return hashlib.sha256(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()).hexdigest()


def oracle_layer(wl: mi.Workload, h: dict, tokens=None, routed_scaling=None, **kw):
    rs = wl.routed_scaling if routed_scaling is None else routed_scaling
    return oracle.moe_layer(h["x"], h["logits"], wl.k, h["w_gate"], h["s_gate"], h["w_up"], h["s_up"],
                            h["w_down"], h["s_down"], rs, tokens=tokens, **kw)
