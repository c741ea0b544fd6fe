"""Seeded synthetic inputs for the routed-MoE FP8 blockwise prefill path.

This module only draws inputs.  It holds none of the path's arithmetic
(routing, activation quantisation, expert FFN, combine) and imports neither
the oracle nor the CUDA library; both sides take their inputs from here.

Workloads (the pages measure real GLM checkpoints, which are not available;
these synthetic workloads stand in for them, with the shapes and value
distributions stated in the workload list of the benchmark specification):

  tiny    T=64    H=256  E=8   k=2 I=128   x~N(0,1)              logits~N(0,1)           rs=1.0
  small   T=1024  H=2048 E=64  k=8 I=512   x~N(0,1)              logits~U[0,1)           rs=2.5
  glm     T=4096  H=5120 E=256 k=8 I=1536  x~N(0,1), 0.1% of      logits Zipf(1.1)        rs=1.0
                                           tokens scaled x100     popularity (Gumbel-top-k)
  non128  T=2048  H=5120 E=160 k=8 I=192   x~N(0,1)              logits~N(0,1), 20% of   rs=1.0
                                                                  experts get -1e4
  long    T=16384 H=6144 E=256 k=8 I=2048  x~Student-t(3)         logits Zipf(1.1)        rs=1.0

Expert weights, every workload: W ~ N(0, 0.02^2) in FP32, stored as E4M3
codes with one FP32 scale per 128x128 block (partial blocks at the edges),
s = amax/448, codes = E4M3(W/s) via torch's float8_e4m3fn conversion.  This
is input preparation (the checkpoint format), not a step of the path.

Every tensor draws from its own torch generator seeded with
hash(seed, tensor-name), so tensors are reproducible independently of one
another for a given device.  CPU and CUDA generators give different streams:
a test that compares two implementations hands both the same tensors.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import torch

FP8_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    routed_scaling: float
    x_dist: str
    logit_dist: str

    @property
    def Ip(self) -> int:
        return ((self.I + 127) // 128) * 128

    @property
    def GH(self) -> int:
        return self.H // 128

    @property
    def GI(self) -> int:
        return (self.I + 127) // 128

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 8, 2, 128, 1.0, "normal", "normal"),
    "small": Workload("small", 1024, 2048, 64, 8, 512, 2.5, "normal", "uniform"),
    "glm": Workload("glm", 4096, 5120, 256, 8, 1536, 1.0, "normal_outliers", "zipf"),
    "non128": Workload("non128", 2048, 5120, 160, 8, 192, 1.0, "normal", "normal_masked"),
    "long": Workload("long", 16384, 6144, 256, 8, 2048, 1.0, "student_t3", "zipf"),
    # GLM widths with 64 experts (1.5 GB of weights): the case detailed
    # profiler captures run on (larger than L2, a few GB on the device)
    "glm64": Workload("glm64", 2048, 5120, 64, 8, 1536, 1.0, "normal_outliers", "zipf"),
    # the long prefill's widths and rows with 32 experts (1.2 GB of weights):
    # the case its DRAM traffic is captured on, scaled to the full layer
    "long32": Workload("long32", 16384, 6144, 32, 8, 2048, 1.0, "student_t3", "zipf"),
}


def _seed(seed: int, name: str) -> int:
    h = hashlib.sha256(f"{seed}:{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed(seed, name))
    return g


def outlier_tokens(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Indices of the tokens scaled x100 in the outlier workload (CPU, sorted)."""
    if wl.x_dist != "normal_outliers":
        return torch.zeros(0, dtype=torch.int64)
    n = int(round(0.001 * wl.T))
    g = generator(seed, "x.outliers", "cpu")
    return torch.randperm(wl.T, generator=g)[:n].sort().values


def masked_experts(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Experts that receive -1e4 on every logit in the masked workload (CPU)."""
    if wl.logit_dist != "normal_masked":
        return torch.zeros(0, dtype=torch.int64)
    n = int(round(0.2 * wl.E))
    g = generator(seed, "logits.mask", "cpu")
    return torch.randperm(wl.E, generator=g)[:n].sort().values


def make_x(wl: Workload, seed: int = 0, device="cpu", T: int | None = None) -> torch.Tensor:
    T = wl.T if T is None else T
    g = generator(seed, "x", device)
    if wl.x_dist in ("normal", "normal_outliers"):
        x = torch.randn((T, wl.H), generator=g, device=device, dtype=torch.float32)
        if wl.x_dist == "normal_outliers":
            idx = outlier_tokens(wl.with_(T=T), seed).to(device)
            x[idx] *= 100.0
    elif wl.x_dist == "student_t3":
        z = torch.randn((T, wl.H), generator=g, device=device, dtype=torch.float32)
        c = torch.zeros_like(z)
        for _ in range(3):
            n = torch.randn((T, wl.H), generator=g, device=device, dtype=torch.float32)
            c += n * n
        x = z / torch.sqrt(c / 3.0)
    else:
        raise ValueError(wl.x_dist)
    return x.to(torch.bfloat16)


def make_logits(wl: Workload, seed: int = 0, device="cpu", T: int | None = None) -> torch.Tensor:
    T = wl.T if T is None else T
    g = generator(seed, "logits", device)
    if wl.logit_dist == "normal":
        return torch.randn((T, wl.E), generator=g, device=device, dtype=torch.float32)
    if wl.logit_dist == "uniform":
        return torch.rand((T, wl.E), generator=g, device=device, dtype=torch.float32)
    if wl.logit_dist == "normal_masked":
        lg = torch.randn((T, wl.E), generator=g, device=device, dtype=torch.float32)
        lg[:, masked_experts(wl, seed).to(device)] += -1.0e4
        return lg
    if wl.logit_dist == "zipf":
        # Gumbel-top-k over log popularity selects experts with probability
        # proportional to the Zipf(1.1) popularity, without replacement.
        gp = generator(seed, "logits.perm", "cpu")
        perm = torch.randperm(wl.E, generator=gp)
        rank = torch.empty(wl.E, dtype=torch.float32)
        rank[perm] = torch.arange(1, wl.E + 1, dtype=torch.float32)
        logz = (-1.1 * torch.log(rank)).to(device)
        u = torch.rand((T, wl.E), generator=g, device=device, dtype=torch.float32)
        u = u.clamp_min(torch.finfo(torch.float32).tiny)
        gumbel = -torch.log(-torch.log(u))
        return gumbel + logz
    raise ValueError(wl.logit_dist)


def _blockwise_fp8(W: torch.Tensor):
    """W [n_e, R, C] FP32 -> codes uint8 [n_e,R,C], scales [n_e,ceil(R/128),ceil(C/128)]."""
    n_e, R, C = W.shape
    Rb, Cb = (R + 127) // 128, (C + 127) // 128
    Wp = torch.zeros((n_e, Rb * 128, Cb * 128), dtype=W.dtype, device=W.device)
    Wp[:, :R, :C] = W
    amax = Wp.abs().view(n_e, Rb, 128, Cb, 128).amax(dim=(2, 4))
    s = amax / FP8_MAX
    s = torch.where(s == 0, torch.ones_like(s), s)
    q = Wp / s.repeat_interleave(128, 1).repeat_interleave(128, 2)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8)[:, :R, :C].contiguous()
    return codes, s.contiguous()


def make_weights(wl: Workload, seed: int = 0, device="cpu", experts_per_chunk: int | None = None):
    """Returns dict w_gate, w_up [E,I,H] u8; w_down [E,H,I] u8; s_gate, s_up
    [E,ceil(I/128),H/128] f32; s_down [E,H/128,ceil(I/128)] f32."""
    E, I, H = wl.E, wl.I, wl.H
    if experts_per_chunk is None:
        experts_per_chunk = max(1, (1 << 27) // (I * H))
    out = {}
    for name, (R, C) in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I))):
        g = generator(seed, f"w_{name}", device)
        codes = torch.empty((E, R, C), dtype=torch.uint8, device=device)
        scales = torch.empty((E, (R + 127) // 128, (C + 127) // 128), dtype=torch.float32, device=device)
        for e0 in range(0, E, experts_per_chunk):
            e1 = min(E, e0 + experts_per_chunk)
            W = torch.randn((e1 - e0, R, C), generator=g, device=device, dtype=torch.float32) * 0.02
            c, s = _blockwise_fp8(W)
            codes[e0:e1] = c
            scales[e0:e1] = s
            del W, c, s
        out[f"w_{name}"] = codes
        out[f"s_{name}"] = scales
    return out


def _mx_fp8(W: torch.Tensor):
    """W [n_e, R, C] FP32 (C % 32 == 0) -> MXFP8: codes uint8 [n_e,R,C] and
    one UE8M0 scale byte per (row, 32 columns) [n_e,R,C/32]: shared exponent
    floor(log2(amax)) - 8, element = float8_e4m3fn(W / 2^se) after clamping to
    +-448.  Input preparation (the checkpoint format), not a step of the path."""
    n_e, R, C = W.shape
    blk = W.view(n_e, R, C // 32, 32)
    amax = blk.abs().amax(dim=-1)
    _, ex = torch.frexp(amax)
    se = torch.where(amax == 0, torch.full_like(ex, -127), (ex - 9).clamp(-127, 127))
    q = (blk * torch.ldexp(torch.ones_like(amax), -se)[..., None]).clamp(-FP8_MAX, FP8_MAX)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8).view(n_e, R, C).contiguous()
    return codes, (se + 127).to(torch.uint8).contiguous()


def make_weights_mx(wl: Workload, seed: int = 0, device="cpu", experts_per_chunk: int | None = None):
    """The weights of make_weights (the same FP32 draws) stored as MXFP8:
    w_gate, w_up [E,I,H] u8 with s_gate, s_up [E,I,H/32] u8 (UE8M0);
    w_down [E,H,I] u8 with s_down [E,H,I/32] u8."""
    E, I, H = wl.E, wl.I, wl.H
    assert I % 32 == 0 and H % 32 == 0
    if experts_per_chunk is None:
        experts_per_chunk = max(1, (1 << 27) // (I * H))
    out = {}
    for name, (R, C) in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I))):
        g = generator(seed, f"w_{name}", device)
        codes = torch.empty((E, R, C), dtype=torch.uint8, device=device)
        scales = torch.empty((E, R, C // 32), dtype=torch.uint8, device=device)
        for e0 in range(0, E, experts_per_chunk):
            e1 = min(E, e0 + experts_per_chunk)
            W = torch.randn((e1 - e0, R, C), generator=g, device=device, dtype=torch.float32) * 0.02
            c, sc = _mx_fp8(W)
            codes[e0:e1] = c
            scales[e0:e1] = sc
            del W, c, sc
        out[f"w_{name}"] = codes
        out[f"s_{name}"] = scales
    return out


def make_inputs_mx(wl: Workload | str, seed: int = 0, device="cpu", T: int | None = None):
    """All inputs of one MXFP8 layer call (x and logits as make_inputs)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    d = {"x": make_x(wl, seed, device, T), "logits": make_logits(wl, seed, device, T)}
    d.update(make_weights_mx(wl, seed, device))
    return d


def make_inputs(wl: Workload | str, seed: int = 0, device="cpu", T: int | None = None):
    """All inputs of one layer call: x, logits, weights and scales."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    d = {"x": make_x(wl, seed, device, T), "logits": make_logits(wl, seed, device, T)}
    d.update(make_weights(wl, seed, device))
    return d


def sample_tokens(wl: Workload, ids: torch.Tensor, n_random: int = 256, seed: int = 0) -> torch.Tensor:
    """Deterministic token sample for sampled parity at full size: every
    outlier token, n_random seeded tokens, and one token routed to the most
    and one to the least loaded active expert.  ids: [T,k] routing (CPU)."""
    T = ids.shape[0]
    picks = [outlier_tokens(wl.with_(T=T), seed)]
    g = generator(seed, "sample", "cpu")
    picks.append(torch.randperm(T, generator=g)[: min(n_random, T)])
    flat = ids.reshape(-1)
    valid = flat[flat >= 0]
    if valid.numel():
        cnt = torch.bincount(valid.long(), minlength=wl.E)
        active = (cnt > 0).nonzero().flatten()
        for e in (int(cnt.argmax()), int(active[cnt[active].argmin()])):
            tok = (ids == e).any(dim=1).nonzero().flatten()
            picks.append(tok[:1])
    return torch.unique(torch.cat(picks).long()).sort().values


def flops_per_layer(wl: Workload, P: int | None = None) -> float:
    P = wl.T * wl.k if P is None else P
    return 6.0 * P * wl.I * wl.H


def algorithmic_bytes(wl: Workload, active_experts: int) -> float:
    """Weights of active experts once, their scales, x, logits, FP32 out."""
    w = 3.0 * wl.I * wl.H * active_experts
    s = 4.0 * active_experts * 3 * wl.GI * wl.GH
    return w + s + wl.T * wl.H * 2 + wl.T * wl.E * 4 + wl.T * wl.H * 4


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_inputs_mx", "make_x", "make_logits", "make_weights",
           "make_weights_mx",
           "outlier_tokens", "masked_experts", "sample_tokens", "flops_per_layer",
           "algorithmic_bytes", "generator", "ceil_div", "math"]
