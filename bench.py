"""Benchmark of the routed-MoE FP8 blockwise (W8A8) prefill layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference] [--workload glm]

One step = one whole layer call (moe_route_quant, moe_grouped_ffn,
moe_combine) over one batch of T tokens, inputs resident in HBM.  Workload:
the GLM-class layer (T=4096, H=5120, 256 experts, top-8, I=1536, 0.1 %
outlier tokens x100, Zipf(1.1) routing), the configuration the throughput
target is stated on.  Multi-GPU (torchrun): every rank runs its own batch on
its own replica of the weights (weak scaling, no collective on the data
path); the timed region is bracketed by barriers and the time is the max
over ranks.

Rank 0 prints one JSON line.  Besides the contract keys it carries:
  roofline      the dominant kernel (the gate/up grouped GEMM), achieved
                algorithmic bytes / its event-timed duration vs measured HBM
                copy bandwidth;
  cpu_baseline  the oracle (plain C, FP64) timed on a bounded token sample
                on this host's cores;
  e2e           the same metric with host buffers: every step copies its
                x and logits from pinned host memory and its FP32 output
                back, pipelined over two layer plans (copy-in, compute and
                copy-out streams overlap); e2e_serial does the same one step
                after the other;
  stages        per-launch-group milliseconds from CUDA events;
  clocks        nvidia-smi samples taken during the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_inputs as mi  # noqa: E402

METRIC = "routed-MoE prefill tokens/s per layer; grouped-GEMM % of B200 FP8 peak"
# kernels of libfp8moe per layer call: route_topk (+ quantiser), route_rank,
# route_scatter, gather_rows, grouped_gemm<0>, grouped_gemm<1>, combine
LAUNCHES_PER_LAYER = 7
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append({"sm": float(f[2]), "max": float(f[3]), "power": float(f[4]),
                             "hw": f[6], "hw_thermal": f[7], "sw_thermal": f[8], "sw_power": f[9]})
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                            ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 200] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun sets RANK/LOCAL_RANK/WORLD_SIZE).  The
    process group carries only barriers and the max of one timing scalar:
    every rank runs its own batch on its own replica of the weights."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, v: float, device="cuda") -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (and weight replica) from its own seed."""
    return rank


def whole_job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step_max: float) -> float:
    """Weak scaling: every rank processes tokens_per_rank per step; the job's
    step time is the slowest rank's."""
    return world * tokens_per_rank / (ms_per_step_max / 1e3)


def kernel_source_sha256() -> str:
    import hashlib

    m = hashlib.sha256()
    for f in ("grouped_ffn.cu", "sm100.cuh"):
        m.update(open(os.path.join(ROOT, "fp8_blockwise_routed_b200", "csrc", f), "rb").read())
    return m.hexdigest()


def recorded_traffic(key: str):
    """DRAM bytes per launch from the committed ncu record, or None when the
    record is missing or the kernel source changed since it was taken."""
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(prof):
        return None
    rec = json.load(open(prof))
    if rec.get("kernel_source_sha256") != kernel_source_sha256():
        return None
    return rec.get(key)


def gateup_alg_bytes(wl, active: int, P: int) -> float:
    """Algorithmic bytes of one gate/up launch: gate+up FP8 weights of the
    active experts and their block scales, the activation codes and scales
    once, the intermediate codes and scales written."""
    return (2.0 * wl.I * wl.H * active + 2 * 4.0 * active * wl.GI * wl.GH
            + wl.T * wl.H + 4.0 * wl.T * wl.GH + P * wl.Ip + 4.0 * P * wl.GI)


def cpu_baseline(wl, d, budget_tokens: int | None = None, seconds: float = 20.0, mx: bool = False):
    """The oracle as it stands (plain C, FP64, OpenMP) on a seeded token
    sample of the same workload (sized to about ``seconds`` of work), timed
    on the host; mx: the MXFP8 variant's oracle on MX inputs.  Returns
    tokens/s."""
    import oracle

    g = mi.generator(0, "cpu_baseline", "cpu")
    perm = torch.randperm(wl.T, generator=g)
    W = [d[k].cpu() for k in ("w_gate", "s_gate", "w_up", "s_up", "w_down", "s_down")]
    xs, ls = d["x"].cpu(), d["logits"].cpu()
    oracle.build()

    def run(n):
        toks = perm[:n].sort().values
        t0 = time.perf_counter()
        (oracle.mx_moe_layer if mx else oracle.moe_layer)(xs[toks], ls[toks], wl.k, *W, wl.routed_scaling)
        return time.perf_counter() - t0

    if budget_tokens:
        n = budget_tokens
    else:  # size the sample to the requested oracle work (a 16-token probe underestimates the rate)
        probe = min(16, wl.T)
        n = max(probe, min(wl.T, int(seconds * probe / max(run(probe), 1e-6))))
    dt = run(n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} seeded tokens of the {wl.name} workload ({'MX ' if mx else ''}quantise, route, FFN, "
                      f"combine), {dt:.1f} s"}


def run_reference(args, wl):
    """The oracle timed as the reference arm: each step evaluates a bounded
    seeded sample of the workload's tokens on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    # the same seeded inputs as the GPU arm when a GPU is present (drawn
    # there in seconds, then copied to the host); only the oracle's
    # evaluation on the host cores is timed
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = {key: v.cpu() for key, v in mi.make_inputs(wl, rank_seed(0), gen_dev).items()}
    if gen_dev == "cuda":
        torch.cuda.empty_cache()
    n = 32  # tokens per step: about a third of a second of oracle work on 16 cores
    W = [d[k] for k in ("w_gate", "s_gate", "w_up", "s_up", "w_down", "s_down")]
    oracle.build()

    def step(i):
        g = mi.generator(i, "reference_sample", "cpu")
        toks = torch.randperm(wl.T, generator=g)[:n].sort().values
        oracle.moe_layer(d["x"][toks], d["logits"][toks], wl.k, *W, wl.routed_scaling)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} seeded tokens per step of the {wl.name} workload"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class E2EPipeline:
    """Host -> device -> host loop over layer plans with double-buffered
    inputs: a copy-in stream, the compute stream and a copy-out stream,
    ordered by events so that a plan's inputs are overwritten only after its
    previous launch has read them and its output only after it was copied
    out."""

    def __init__(self, plans, x_ins, lg_ins, x_h, lg_h, out_hs):
        self.plans, self.x_ins, self.lg_ins = plans, x_ins, lg_ins
        self.x_h, self.lg_h, self.out_hs = x_h, lg_h, out_hs
        self.h2d, self.comp, self.d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        n = len(plans)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]
        self.ev_comp = [torch.cuda.Event() for _ in range(n)]
        self.ev_out = [torch.cuda.Event() for _ in range(n)]

    def run(self, steps: int) -> float:
        """Runs `steps` steps; returns their device time in ms (first copy in
        to last copy out)."""
        n = len(self.plans)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(self.h2d)
        for i in range(steps):
            b = i % n
            used = i >= n
            if used:
                self.h2d.wait_event(self.ev_comp[b])  # plan b has read its previous inputs
            with torch.cuda.stream(self.h2d):
                self.x_ins[b].copy_(self.x_h, non_blocking=True)
                self.lg_ins[b].copy_(self.lg_h, non_blocking=True)
                self.ev_in[b].record(self.h2d)
            self.comp.wait_event(self.ev_in[b])
            if used:
                self.comp.wait_event(self.ev_out[b])  # its previous output has been copied out
            self.plans[b].launch(self.comp)
            self.ev_comp[b].record(self.comp)
            self.d2h.wait_event(self.ev_comp[b])
            with torch.cuda.stream(self.d2h):
                self.out_hs[b].copy_(self.plans[b].out, non_blocking=True)
                self.ev_out[b].record(self.d2h)
        t1.record(self.d2h)
        t1.synchronize()
        return t0.elapsed_time(t1)


def gemm_roofline_s(wl, P: int, active: int, pk) -> float:
    """max(FLOPs / FP8 peak, weight and scale bytes / HBM) of the two grouped
    GEMMs (real I, valid pairs, active experts' weights once)."""
    fp8_peak = 2.0 * pk["bf16_tflops"]  # nominal FP8:BF16 ratio 2 on the measured BF16 peak
    wbytes = mi.algorithmic_bytes(wl, active) - wl.T * wl.H * 4 - wl.T * wl.H * 2 - wl.T * wl.E * 4
    return max(mi.flops_per_layer(wl, P) / (fp8_peak * 1e12), wbytes / (pk["hbm_gbs"] * 1e9))


def measure_workload(wl, steps: int, warmup: int, seed: int, pk, with_cpu: bool):
    """One workload through the graph-launched layer: device time per step
    over `steps` replays, per-stage means from the graph's event nodes, the
    grouped GEMMs against their roofline, and the oracle on a ~3 s token
    sample of the same inputs."""
    import fp8_blockwise_routed_b200 as fm

    d = mi.make_inputs(wl, seed=seed, device="cuda")
    x_in = d["x"].clone()
    lg_in = d["logits"].clone()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    plan = fm.LayerPlan(x_in, lg_in, wl.k, d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"],
                        d["s_down"], wl.routed_scaling, stage_events=ev)
    for _ in range(warmup):
        plan.launch()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for _ in range(steps):
        plan.launch()
    t1.record(s)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    spans = {"route_quant": (0, 1), "gather": (1, 2), "gemm_gateup": (2, 3), "gemm_down": (3, 4),
             "combine": (4, 5)}
    acc = {n: [] for n in spans}
    for _ in range(max(steps, 5)):
        plan.launch()
        torch.cuda.synchronize()
        for n, (a, b) in spans.items():
            acc[n].append(ev[a].elapsed_time(ev[b]))
    st = {n: statistics.mean(v) for n, v in acc.items()}
    status = plan.device_status()
    ws = plan.ws
    T, H, I, E, k = plan.shape
    # expert offsets live in the plan's workspace; the layer's own view gives them
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                         wl.routed_scaling, wl.T)
    layer.forward(d["x"], d["logits"])
    torch.cuda.synchronize()
    off = layer.offsets.cpu()
    P = int(off[-1])
    active = int(((off[1:] - off[:-1]) > 0).sum())
    gemm_s = (st["gemm_gateup"] + st["gemm_down"]) / 1e3
    flops = mi.flops_per_layer(wl, P)
    roof = gemm_roofline_s(wl, P, active, pk)
    res = {"ms_per_step": ms, "tokens_per_s": wl.T / (ms / 1e3), "stages_ms": st,
           "gemm_tflops": flops / gemm_s / 1e12, "gemm_roofline_ms": roof * 1e3,
           "gemm_frac_roofline": roof / gemm_s, "pairs": P, "active_experts": active,
           "device_status": status | layer.device_status()}
    if with_cpu:
        res["cpu_oracle"] = cpu_baseline(wl, d, seconds=3.0)
    plan.close()
    del plan, layer, d, x_in, lg_in, ws
    torch.cuda.empty_cache()
    return res


def measure_workload_mx(wl, steps: int, warmup: int, seed: int, pk, with_cpu: bool):
    """The MXFP8 variant of the layer on one workload (the same FP32 weight
    draws, stored as MX E4M3 with UE8M0 scales per 32 values): device time per
    step of RoutedMoEMX.forward (4 ABI calls, no graph), per-stage means, the
    grouped GEMMs against the same roofline as the 128x128-block path, and
    the MX oracle on a ~3 s token sample."""
    import fp8_blockwise_routed_b200 as fm

    d = mi.make_inputs_mx(wl, seed=seed, device="cuda")
    layer = fm.RoutedMoEMX(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                           wl.routed_scaling, wl.T)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in ev:
        e.record()
    for _ in range(warmup):
        layer.forward(d["x"], d["logits"])
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for _ in range(steps):
        layer.forward(d["x"], d["logits"])
    t1.record(s)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    spans = {"quant_route": (0, 1), "gather": (1, 2), "gemm_gateup": (2, 3), "gemm_down": (3, 4),
             "combine": (4, 5)}
    acc = {n: [] for n in spans}
    for _ in range(max(steps, 5)):
        layer.forward(d["x"], d["logits"], stage_events=ev)
        torch.cuda.synchronize()
        for n, (a, b) in spans.items():
            acc[n].append(ev[a].elapsed_time(ev[b]))
    st = {n: statistics.mean(v) for n, v in acc.items()}
    off = layer.offsets.cpu()
    P = int(off[-1])
    active = int(((off[1:] - off[:-1]) > 0).sum())
    gemm_s = (st["gemm_gateup"] + st["gemm_down"]) / 1e3
    flops = mi.flops_per_layer(wl, P)
    roof = gemm_roofline_s(wl, P, active, pk)
    res = {"format": "MXFP8 (E4M3, UE8M0 scale per 32 values)", "ms_per_step": ms,
           "tokens_per_s": wl.T / (ms / 1e3), "stages_ms": st, "gemm_tflops": flops / gemm_s / 1e12,
           "gemm_roofline_ms": roof * 1e3, "gemm_frac_roofline": roof / gemm_s, "pairs": P,
           "active_experts": active, "device_status": layer.device_status()}
    if with_cpu:
        res["cpu_oracle"] = cpu_baseline(wl, d, seconds=3.0, mx=True)
    del layer, d
    torch.cuda.empty_cache()
    return res


def layer_only(wl, n: int, mx: bool = False):
    """The layer of `wl` (seed 0) n times through moe_route_quant,
    moe_grouped_ffn and moe_combine, for profiler captures: each call launches
    route_topk, route_rank, route_scatter, gather_rows, grouped_gemm (gate/up),
    grouped_gemm (down) and combine, in that order.  mx: the MXFP8 variant
    (RoutedMoEMX): quant_mx, route_topk, route_rank, route_scatter, gather_mx,
    grouped_mx (gate/up), grouped_mx (down), combine."""
    import fp8_blockwise_routed_b200 as fm

    if mx:
        d = mi.make_inputs_mx(wl, seed=0, device="cuda")
        cls = fm.RoutedMoEMX
    else:
        d = mi.make_inputs(wl, seed=0, device="cuda")
        cls = fm.RoutedMoE
    layer = cls(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"], wl.k,
                wl.routed_scaling, wl.T)
    for _ in range(n):
        layer.forward(d["x"], d["logits"])
    torch.cuda.synchronize()
    off = layer.offsets.cpu()
    print(json.dumps({"workload": wl.name, "format": "mxfp8" if mx else "fp8 128x128 blocks", "calls": n,
                      "device_status": layer.device_status(),
                      "pairs": int(off[-1]), "active_experts": int(((off[1:] - off[:-1]) > 0).sum())}))


def workload_config(wl):
    return {"workload": f"{wl.name}: T={wl.T} H={wl.H} E={wl.E} top_k={wl.k} I={wl.I} "
                        f"rs={wl.routed_scaling} x={wl.x_dist} logits={wl.logit_dist}",
            "global_batch": wl.T, "parallelism": "data-parallel replicas (one batch per GPU)",
            "l2": "inputs larger than L2: FP8 expert weights read per step exceed 126 MB"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default="glm", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload lines of the other configurations")
    ap.add_argument("--layer-only", type=int, default=0, metavar="N",
                    help="run the workload's layer N times through the separate calls and exit "
                         "(the program profiler captures run)")
    ap.add_argument("--mxfp8", action="store_true", help="with --layer-only: the MXFP8 variant's layer")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = mi.WORKLOADS[args.workload]
    if args.layer_only:
        layer_only(wl, args.layer_only, mx=args.mxfp8)
        return
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import fp8_blockwise_routed_b200 as fm

    world, rank, local = dist_setup("nccl")
    dev = torch.device("cuda", torch.cuda.current_device())
    d = mi.make_inputs(wl, seed=rank_seed(rank), device=dev)
    layer = fm.RoutedMoE(d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"], d["s_down"],
                         wl.k, wl.routed_scaling, wl.T)
    s = torch.cuda.current_stream()

    # The product path: the layer captured once into a CUDA graph (the C
    # ABI's moe_layer_plan) over resident input buffers, replayed per step.
    x_in = torch.empty_like(d["x"])
    lg_in = torch.empty_like(d["logits"])
    x_in.copy_(d["x"])
    lg_in.copy_(d["logits"])
    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    plan = fm.LayerPlan(x_in, lg_in, wl.k, d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"],
                        d["s_down"], wl.routed_scaling, stage_events=stage_ev)
    for _ in range(args.warmup):
        layer.forward(d["x"], d["logits"])
        plan.launch()
    torch.cuda.synchronize()
    if layer.device_status() != 0 or plan.device_status() != 0:
        raise RuntimeError("device status reported a fault during warm-up")
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for i in range(args.steps):
        plan.launch()
    t1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms_total = max_over_ranks(world, t0.elapsed_time(t1))
    ms_step = ms_total / args.steps
    # the graph's event nodes hold the last timed replay's marks
    spans = {"route_quant": (0, 1), "gather": (1, 2), "gemm_gateup": (2, 3), "gemm_down": (3, 4),
             "combine": (4, 5)}
    last_ms = {n: stage_ev[a].elapsed_time(stage_ev[b]) for n, (a, b) in spans.items()}
    status = plan.device_status()

    # Per-stage averages from the events inside the graph (one launch at a
    # time, after the timed region), and the same layer through the three
    # separate calls.
    acc = {n: [] for n in spans}
    for _ in range(args.steps):
        plan.launch()
        torch.cuda.synchronize()
        for n, (a, b) in spans.items():
            acc[n].append(stage_ev[a].elapsed_time(stage_ev[b]))
    stage_ms = {n: statistics.mean(v) for n, v in acc.items()}
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    c0.record(s)
    for _ in range(args.steps):
        layer.forward(d["x"], d["logits"])
    c1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    ms_calls = max_over_ranks(world, c0.elapsed_time(c1)) / args.steps
    status |= layer.device_status()

    # roofline of the dominant kernel
    pk = peaks()
    off = layer.offsets.cpu()
    P = int(off[-1])
    active = int(((off[1:] - off[:-1]) > 0).sum())
    gu_bytes = gateup_alg_bytes(wl, active, P)
    gu_s = last_ms["gemm_gateup"] / 1e3
    achieved = gu_bytes / gu_s / 1e9
    flops = mi.flops_per_layer(wl, P)
    gemm_s = (stage_ms["gemm_gateup"] + stage_ms["gemm_down"]) / 1e3
    fp8_peak = 2.0 * pk["bf16_tflops"]  # nominal FP8:BF16 ratio 2 on the measured BF16 peak
    roof_s = gemm_roofline_s(wl, P, active, pk)
    traffic = recorded_traffic(f"gemm_gateup/{wl.name}")

    # end to end through the C ABI with host buffers
    x_h = d["x"].cpu().pin_memory()
    lg_h = d["logits"].cpu().pin_memory()
    out_h = torch.empty((wl.T, wl.H), dtype=torch.float32).pin_memory()
    for _ in range(2):
        x_in.copy_(x_h, non_blocking=True)
        lg_in.copy_(lg_h, non_blocking=True)
        out_h.copy_(plan.launch(), non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        x_in.copy_(x_h, non_blocking=True)
        lg_in.copy_(lg_h, non_blocking=True)
        out_h.copy_(plan.launch(), non_blocking=True)
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    e2e_serial_ms = max_over_ranks(world, e0.elapsed_time(e1)) / args.steps

    # The same, pipelined as a serving loop runs it: two plans over
    # double-buffered inputs; step i+1's inputs are copied in while step i
    # computes and step i-1's output is copied out (three streams, ordered
    # by events).  Every step still copies its own inputs and result.
    x_in2 = torch.empty_like(d["x"])
    lg_in2 = torch.empty_like(d["logits"])
    plan2 = fm.LayerPlan(x_in2, lg_in2, wl.k, d["w_gate"], d["s_gate"], d["w_up"], d["s_up"], d["w_down"],
                         d["s_down"], wl.routed_scaling)
    out_h2 = torch.empty_like(out_h).pin_memory()
    pipe = E2EPipeline([plan, plan2], [x_in, x_in2], [lg_in, lg_in2], x_h, lg_h, [out_h, out_h2])
    pipe.run(2)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(world, pipe.run(args.steps)) / args.steps
    status |= plan2.device_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, d)

    # every other workload on this rank's GPU, one after the other (the
    # headline's buffers released first)
    configs = {}
    if not args.no_configs:
        plan2.close()
        del pipe, plan2, x_in2, lg_in2
        torch.cuda.empty_cache()
        for name in ("tiny", "small", "non128", "long"):
            if name == wl.name:
                continue
            configs[name] = measure_workload(mi.WORKLOADS[name], args.steps, args.warmup, rank_seed(rank), pk,
                                             with_cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))
        configs[wl.name + "_mxfp8"] = measure_workload_mx(
            wl, args.steps, args.warmup, rank_seed(rank), pk,
            with_cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": whole_job_tokens_per_s(world, wl.T, ms_step),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "fp8e4m3 (fp32 accumulate)",
            "data": "synthetic (seeded; no checkpoint)",
            "config": workload_config(wl),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                         "kernel": "grouped_gemm_kernel<gate/up>",
                         "alg_bytes_per_launch": gu_bytes, "peak_source": pk["source"]},
            "grouped_gemm": {"ms": gemm_s * 1e3, "tflops": flops / gemm_s / 1e12,
                             "frac_fp8_peak": flops / gemm_s / 1e12 / fp8_peak,
                             "fp8_peak_tflops": fp8_peak, "roofline_ms": roof_s * 1e3,
                             "frac_roofline": roof_s / gemm_s},
            "stages_ms": stage_ms,
            "stages_ms_last_timed_step": last_ms,
            "ms_per_step_three_calls": ms_calls,
            "e2e_serial": {"value": whole_job_tokens_per_s(world, wl.T, e2e_serial_ms), "unit": "tokens/s",
                           "ms_per_step": e2e_serial_ms},
            "e2e": {"value": whole_job_tokens_per_s(world, wl.T, e2e_ms), "unit": "tokens/s",
                    "pipelined": "H2D of step i+1 and D2H of step i-1 overlap step i's compute",
                    "h2d_bytes_per_step": int(x_h.numel() * 2 + lg_h.numel() * 4),
                    "d2h_bytes_per_step": int(out_h.numel() * 4), "ms_per_step": e2e_ms},
            "gpu_launches": LAUNCHES_PER_LAYER * args.steps,
            "device_status": status,
            "active_experts": active,
            "pairs": P,
        }
        if cpu:
            line["cpu_baseline"] = cpu
        if clocks:
            line["clocks"] = clocks
        if configs:
            configs[wl.name] = {"ms_per_step": ms_step, "tokens_per_s": wl.T / (ms_step / 1e3),
                                "stages_ms": stage_ms, "gemm_tflops": flops / gemm_s / 1e12,
                                "gemm_roofline_ms": roof_s * 1e3, "gemm_frac_roofline": roof_s / gemm_s,
                                "pairs": P, "active_experts": active, "device_status": status}
            if cpu:
                configs[wl.name]["cpu_oracle"] = cpu
            line["configs"] = configs
        print(json.dumps(line), flush=True)
    plan.close()
    if args.no_configs:
        plan2.close()
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
