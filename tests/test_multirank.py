"""The multi-rank path of the benchmark on CPU: two gloo ranks (no GPU).
Every rank processes its own batch (weak scaling, no data-path collective);
the timed region is bracketed by barriers and the job's step time is the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
import moe_inputs as mi


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (world, rank)
    # each rank draws a different batch of the same workload
    wl = mi.WORKLOADS["tiny"]
    x = mi.make_x(wl, bench.rank_seed(r), "cpu")
    digest = float(x.float().sum())
    bench.barrier(w)
    my_ms = 1.0 + r  # rank 1 is the slow one
    mx = bench.max_over_ranks(w, my_ms, device="cpu")
    all_digests = [torch.zeros(1, dtype=torch.float64) for _ in range(w)]
    torch.distributed.all_gather(all_digests, torch.tensor([digest], dtype=torch.float64))
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    out[r] = (mx, [float(d) for d in all_digests])


def test_two_gloo_ranks_max_time_and_distinct_batches():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 2.0           # max over ranks
    d = out[0][1]
    assert d[0] != d[1]                             # different batches per rank
    assert bench.whole_job_tokens_per_s(2, 4096, 2.0) == pytest.approx(2 * 4096 / 2e-3)


def test_single_rank_no_process_group():
    os.environ.pop("WORLD_SIZE", None)
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (1, 0)
    assert bench.max_over_ranks(1, 3.5, device="cpu") == 3.5


# ---- the expert-parallel row exchange (point-to-point; gloo on CPU here,
# ---- NCCL over NVLink on GPUs)

_COUNTS = [[2, 0, 3], [1, 4, 0], [0, 2, 5]]  # rows rank src sends to rank dst


def _exchange_worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    bench.dist_setup("gloo")
    from fp8_blockwise_routed_b200 import ep
    send_counts = _COUNTS[rank]
    recv_counts = [_COUNTS[src][rank] for src in range(world)]
    H = 4
    rows = []
    for dst in range(world):
        for i in range(send_counts[dst]):
            rows.append([rank * 1000 + dst * 100 + i + 0.25 * c for c in range(H)])
    send = torch.tensor(rows, dtype=torch.float32) if rows else torch.zeros((0, H))
    recv = torch.full((sum(recv_counts), H), -1.0)
    ep.exchange_rows(send, send_counts, recv, recv_counts)
    bench.barrier(world)
    torch.distributed.destroy_process_group()
    out[rank] = recv.tolist()


def test_expert_parallel_row_exchange_three_gloo_ranks():
    world = 3
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_exchange_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for dst in range(world):
        want = [[src * 1000 + dst * 100 + i + 0.25 * c for c in range(4)]
                for src in range(world) for i in range(_COUNTS[src][dst])]
        assert out[dst] == want
