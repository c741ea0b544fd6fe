"""Expert parallelism across the ranks of a torch.distributed group.

Rank r owns experts [r*E/world, (r+1)*E/world) and is home to tokens
[r*T_home, (r+1)*T_home) with T_home = ceil(T/world).  Every rank runs the
router over all T tokens (the same ids everywhere), computes the pairs of its
own experts with the grouped FFN, and sends each pair's y row to the pair's
home rank; a home rank sums its tokens' k slot rows in slot order.  A row's
bits are therefore those of the single-GPU layer, whatever the sharding
(reading of the pages: one exchange on each side of the expert compute, and
a row's bits independent of how many rows share a call -- "GLM-5.3-Flash
EXL3 on CUDA ...", exactness note).

Every step runs in libfp8moe's kernels (moe_route_quant, moe_ep_plan,
moe_permute, moe_grouped_ffn_rows, moe_combine_rows); the rows move between
ranks through torch.distributed point-to-point operations (NCCL over NVLink
on GPUs; the same code runs on gloo).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (moe_combine_rows, moe_combine_workspace_bytes, moe_ep_plan, moe_ep_plan_workspace_bytes,
               moe_ffn_workspace_bytes, moe_get_device_status, moe_grouped_ffn_rows, moe_permute, moe_route_quant,
               moe_route_workspace_bytes)


def home_tokens(T: int, world: int) -> int:
    return -(-T // world)


def exchange_rows(send: torch.Tensor, send_counts, recv: torch.Tensor, recv_counts, group=None):
    """Rows send[sum(send_counts[:h]) : +send_counts[h]] go to rank h and land,
    on rank h, at recv[sum(recv_counts[:r]) : +recv_counts[r]] (r the sender).
    Both sides derive their counts from the same routing, so they agree."""
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = len(send_counts)
    soff = [0] * (world + 1)
    roff = [0] * (world + 1)
    for i in range(world):
        soff[i + 1] = soff[i] + int(send_counts[i])
        roff[i + 1] = roff[i] + int(recv_counts[i])
    if send_counts[rank]:
        recv[roff[rank]:roff[rank + 1]].copy_(send[soff[rank]:soff[rank + 1]])
    ops = []
    for peer in range(world):
        if peer == rank:
            continue
        if send_counts[peer]:
            ops.append(dist.P2POp(dist.isend, send[soff[peer]:soff[peer + 1]].contiguous(), peer, group))
        if recv_counts[peer]:
            ops.append(dist.P2POp(dist.irecv, recv[roff[peer]:roff[peer + 1]], peer, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


class ExpertParallelMoE:
    """One rank's share of an expert-parallel routed layer.  w_* / s_* hold
    this rank's experts only ([E/world, ...]); ``forward`` takes the full
    batch (x [T, H] BF16, logits [T, E]) and returns the FP32 rows of this
    rank's home tokens."""

    def __init__(self, w_gate, s_gate, w_up, s_up, w_down, s_down, num_experts: int, top_k: int,
                 routed_scaling: float, max_tokens: int, rank: int = 0, world: int = 1, group=None):
        self.w = (w_gate, s_gate, w_up, s_up, w_down, s_down)
        self.E_local, self.I, self.H = w_gate.shape
        self.E = int(num_experts)
        assert self.E == self.E_local * world
        self.k, self.rs = int(top_k), float(routed_scaling)
        self.rank, self.world, self.group = rank, world, group
        T, H, k = int(max_tokens), self.H, self.k
        dev = w_gate.device
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        self.max_tokens = T
        self.codes = torch.empty((T, H), dtype=u8, device=dev)
        self.scales = torch.empty((T, H // 128), dtype=f32, device=dev)
        self.ids = torch.empty((T, k), dtype=i32, device=dev)
        self.tw = torch.empty((T, k), dtype=f32, device=dev)
        self.offsets = torch.empty((self.E + 1,), dtype=i32, device=dev)
        self.sorted = torch.empty((T * k,), dtype=i32, device=dev)
        self.local_ids = torch.empty((T, k), dtype=i32, device=dev)
        self.send_rows = torch.empty((T * k,), dtype=i32, device=dev)
        self.recv_rows = torch.empty((home_tokens(T, world), k), dtype=i32, device=dev)
        self.offs_oh = torch.empty((world * world + 1,), dtype=i32, device=dev)
        self.offs_ho = torch.empty((world * world + 1,), dtype=i32, device=dev)
        self.offsets_local = torch.empty((self.E_local + 1,), dtype=i32, device=dev)
        self.sorted_local = torch.empty((T * k,), dtype=i32, device=dev)
        self.send = torch.empty((T * k, H), dtype=f32, device=dev)
        self.recv = torch.empty((home_tokens(T, world) * k, H), dtype=f32, device=dev)
        self.out = torch.empty((home_tokens(T, world), H), dtype=f32, device=dev)
        self.ws_route = torch.empty((moe_route_workspace_bytes(T, self.E, k),), dtype=u8, device=dev)
        self.ws_perm = torch.empty((moe_route_workspace_bytes(T, self.E_local, k),), dtype=u8, device=dev)
        self.ws_ep = torch.empty((moe_ep_plan_workspace_bytes(T, k, world),), dtype=u8, device=dev)
        self.ws_ffn = torch.empty((moe_ffn_workspace_bytes(T, H, self.I, self.E_local, k),), dtype=u8, device=dev)
        self.ws_comb = torch.empty((moe_combine_workspace_bytes(),), dtype=u8, device=dev)
        # the (owner, home) count tables are copied into pinned host memory
        # as soon as the plan kernel has written them; the host waits for
        # that copy (an event), not for the grouped FFN enqueued behind it
        pin = dev.type == "cuda"
        self._oh_h = torch.empty((world * world + 1,), dtype=i32, pin_memory=pin)
        self._ho_h = torch.empty((world * world + 1,), dtype=i32, pin_memory=pin)
        self._counts_ready = torch.cuda.Event() if pin else None

    def _split(self, oh, ho):
        w, r = self.world, self.rank
        send = [oh[r * w + h + 1] - oh[r * w + h] for h in range(w)]
        recv = [ho[r * w + o + 1] - ho[r * w + o] for o in range(w)]
        return send, recv

    def counts(self, T: int):
        """Rows this rank sends to each home and receives from each owner
        (synchronous read of the device tables)."""
        return self._split(self.offs_oh.cpu().tolist(), self.offs_ho.cpu().tolist())

    def forward(self, x: torch.Tensor, logits: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        k, w, r = self.k, self.world, self.rank
        assert T <= self.max_tokens and logits.shape == (T, self.E)
        T_home = home_tokens(T, w)
        t0, t1 = min(T, r * T_home), min(T, (r + 1) * T_home)
        codes, scales, ids, tw = self.codes[:T], self.scales[:T], self.ids[:T], self.tw[:T]
        local_ids, recv_rows = self.local_ids[:T], self.recv_rows[:T_home]
        moe_route_quant(logits, x, k, ids, tw, self.offsets, self.sorted[:T * k], codes, scales, self.ws_route, stream)
        moe_ep_plan(ids, self.E, w, r, T_home, local_ids, self.send_rows[:T * k], recv_rows, self.offs_oh,
                    self.offs_ho, self.ws_ep, stream)
        if self._counts_ready is not None:
            s = torch.cuda.current_stream() if stream is None else stream
            with torch.cuda.stream(s):
                self._oh_h.copy_(self.offs_oh, non_blocking=True)
                self._ho_h.copy_(self.offs_ho, non_blocking=True)
            self._counts_ready.record(s)
        moe_permute(local_ids, self.E_local, self.offsets_local, self.sorted_local[:T * k], self.ws_perm, stream)
        # The send buffer has a row for every pair (T*k rows, whatever this
        # rank's share turns out to be), so the grouped FFN is enqueued before
        # the counts reach the host and runs while the host reads them.
        moe_grouped_ffn_rows(codes, scales, local_ids, tw, self.offsets_local, self.sorted_local[:T * k], *self.w,
                             self.send[:T * k], self.send_rows[:T * k], self.ws_ffn, stream)
        if self._counts_ready is not None:
            self._counts_ready.synchronize()  # routing and plan done; the FFN may still run
            send_counts, recv_counts = self._split(self._oh_h.tolist(), self._ho_h.tolist())
        else:
            send_counts, recv_counts = self.counts(T)
        exchange_rows(self.send, send_counts, self.recv, recv_counts, self.group)
        out = self.out[:t1 - t0]
        moe_combine_rows(self.recv[:max(sum(recv_counts), 1)], recv_rows[:t1 - t0], self.rs, out, None,
                         self.ws_comb, stream)
        return out

    def device_status(self) -> int:
        return (moe_get_device_status(self.ws_route) | moe_get_device_status(self.ws_ep)
                | moe_get_device_status(self.ws_ffn) | moe_get_device_status(self.ws_comb))
