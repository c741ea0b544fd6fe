"""Brute-force dense evaluator used to pin the oracle (tests only).

Written independently of ``oracle/oracle.c``: it decodes with torch's
``float8_e4m3fn`` type, evaluates EVERY expert for EVERY token with FP64
torch matmuls (no permutation, no gather), selects by a full stable sort of
each logit row, and requantises the intermediate with torch's FP32 divide and
float8 conversion.  Only small shapes are practical.
"""
from __future__ import annotations

import numpy as np
import torch


def decode_table() -> torch.Tensor:
    """E4M3 byte -> FP64 via torch; the two NaN bytes are mapped to signed
    zero, following the NaN-to-signed-zero policy of the page "Exact AVX2 FP8
    arithmetic conversion avoids costly LUT gathers" ("Semantics and scope")."""
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = b.view(torch.float8_e4m3fn).to(torch.float64)
    v[0x7F] = 0.0
    v[0xFF] = -0.0
    return v


def _expand(s: torch.Tensor, R: int, C: int) -> torch.Tensor:
    """Block scales [Rb,Cb] -> per-element [R,C] (each scale covers 128x128)."""
    return s.repeat_interleave(128, 0).repeat_interleave(128, 1)[:R, :C]


def dequant_matrix(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    dec = decode_table()
    R, C = codes.shape
    return dec[codes.long()] * _expand(scales.double(), R, C)


def requant_rows(h32: torch.Tensor):
    """Quantise FP32 rows per 128-column group with torch ops: scale =
    fl32(amax/448) (1 if that is 0), codes = float8(fl32(h/scale)).  Partial
    last group uses its real columns.  Returns FP64 dequantised rows, codes,
    scales.  Non-finite inputs are not supported here."""
    n, I = h32.shape
    G = (I + 127) // 128
    codes = torch.zeros((n, G * 128), dtype=torch.uint8)
    scales = torch.zeros((n, G), dtype=torch.float32)
    deq = torch.zeros((n, I), dtype=torch.float64)
    dec = decode_table()
    for g in range(G):
        c0, c1 = g * 128, min(I, g * 128 + 128)
        blk = h32[:, c0:c1]
        amax = blk.abs().amax(dim=1)
        s = amax / torch.tensor(448.0, dtype=torch.float32)
        s = torch.where(s == 0, torch.ones_like(s), s)
        q = (blk / s[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        codes[:, c0:c1] = q
        scales[:, g] = s
        deq[:, c0:c1] = dec[q.long()] * s[:, None].double()
    return deq, codes, scales


def route_full_sort(logits: torch.Tensor, k: int):
    """Top-k by a full stable sort (value descending, id ascending), skipping
    NaN and -Inf; weights are the FP64 softmax of the selected logits."""
    T, E = logits.shape
    ids = np.full((T, k), -1, np.int32)
    w = np.zeros((T, k), np.float64)
    L = logits.double().numpy()
    for t in range(T):
        row = L[t]
        ok = [e for e in range(E) if not (np.isnan(row[e]) or row[e] == -np.inf)]
        order = sorted(ok, key=lambda e: (-row[e], e))[:k]
        if not order:
            continue
        v = np.array([row[e] for e in order])
        ex = np.exp(v - v.max())
        ids[t, : len(order)] = order
        w[t, : len(order)] = ex / ex.sum()
    return ids, w


def dense_moe(codes, act_scales, logits, k, wg, sg, wu, su, wd, sd, rs):
    """Whole layer, densely.  Returns (out [T,H] FP64, ids, weights,
    h_codes [T,E,Ip]) where h_codes are the requantised intermediates of every
    (token, expert) pair."""
    codes = torch.as_tensor(codes)
    act_scales = torch.as_tensor(act_scales)
    T, H = codes.shape
    E, I, _ = wg.shape
    dec = decode_table()
    xd = dec[codes.long()] * act_scales.double().repeat_interleave(128, 1)
    ids, w = route_full_sort(torch.as_tensor(logits), k)
    O = torch.zeros((E, T, H), dtype=torch.float64)
    Ip = ((I + 127) // 128) * 128
    HC = torch.zeros((T, E, Ip), dtype=torch.uint8)
    for e in range(E):
        G = xd @ dequant_matrix(wg[e], sg[e]).T
        U = xd @ dequant_matrix(wu[e], su[e]).T
        h32 = (G / (1.0 + torch.exp(-G)) * U).to(torch.float32)
        hdq, hc, _ = requant_rows(h32)
        HC[:, e] = hc
        O[e] = hdq @ dequant_matrix(wd[e], sd[e]).T
    out = torch.zeros((T, H), dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            if ids[t, j] >= 0:
                out[t] += w[t, j] * O[ids[t, j], t]
    return (rs * out).numpy(), ids, w, HC.numpy()
