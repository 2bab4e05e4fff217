#!/usr/bin/env python3
"""Benchmark of the recurrent KDA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one ``kda_decode`` call over one batch (default workload
``n32_t1_hv8``: N=32 sequences, T=1 token, HV=8 value heads, K=V=128, fp32
state pool of 64 slots).  A timed region replays, from CUDA graphs, exactly K
calls that rotate over R independent replicas of the inputs and pool whose
combined touched bytes exceed twice the L2 cache, so every call reads its state
from HBM (the pages' cold-L2 graph-replay method).  The regions are enqueued
behind an untimed pre-roll of replays with no host sync in between, so neither
an idle GPU nor a graph-launch gap is counted; each region sits between CUDA
events on the launching stream, the reported time is the median region, with a
device synchronize on both sides of the whole run.  Under torchrun each rank
runs its own batch (weak scaling, no collective on the data path) and the
reported time is the maximum over ranks.

Printed (rank 0, one JSON line): µs per call for the whole job, the achieved
HBM bandwidth of the decode kernel against the measured copy bandwidth
(roofline), the fp64 oracle timed on the host cores (cpu_baseline), the same
metric end to end through the public Python API with pinned host buffers
(e2e), SM clocks sampled during the timed region, and the kernel launch count.

``--impl reference`` times the fp64 oracle instead (on rank 0, host cores).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA decode µs/call and achieved HBM GB/s (% of B200 peak) at N32/T1/HV8"
UNIT = "us/call"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "linear_attention_recurrent_decode_b200", "csrc")
PROFILES = os.path.join(ROOT, "profiles")


# ------------------------------------------------------------------ helpers
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_max(value: float, device=None) -> float:
    """Maximum of ``value`` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling): disjoint seed streams."""
    return base + 100_003 * rank


def kernel_source_hash(names=("kda_decode_kernel.cuh", "kda_decode_api.cu")) -> str:
    """Hash of the source files that define a kernel and its launch (by default
    the decode kernels): a profile taken from other sources is stale."""
    h = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """dram bytes (read + write) per launch from a committed ncu summary under
    profiles/ taken on this workload with the current kernel source; else None."""
    if not os.path.isdir(PROFILES):
        return None
    current = kernel_source_hash()
    for name in sorted(os.listdir(PROFILES)):
        if not name.endswith(".md"):
            continue
        fields = {}
        with open(os.path.join(PROFILES, name)) as f:
            for line in f:
                if line.startswith("- ") and ":" in line:
                    key, val = line[2:].split(":", 1)
                    fields.setdefault(key.strip(), val.strip().strip("`"))
        if fields.get("workload") != workload or fields.get("kernel_source_hash") != current:
            continue
        try:
            return int(fields["dram_bytes_per_launch"])
        except (KeyError, ValueError):
            continue
    return None


def fp32_alu_peak_tflops(sms: int, mhz: float = 1965.0) -> float:
    """fp32 CUDA-core peak: SMs x 128 fp32 FMA lanes (4 sub-partitions x 32)
    x 2 flop per FMA x the SM clock (B200's clocks.max.sm, 1965 MHz)."""
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def prefill_state_flops(w) -> int:
    """Algorithmic flops of the prefill's state recurrence (stage 1) for one
    call: per chunk of Tc tokens and (n, h), U = Ut - W S0 (2 Tc K V), the
    decay D S0 (K V), S = D S0 + Kh^T U (2 K Tc V) and the subtraction (Tc V)."""
    nchunks = (w.T + 63) // 64
    return w.N * w.HV * (4 * w.T * w.K * w.V + nchunks * w.K * w.V + w.T * w.V)


def prefill_output_flops(w) -> int:
    """Algorithmic flops of the prefill's chunk outputs (stage 2, the tensor-core
    kernel) for one call: per chunk of Tc tokens and (n, h), Qt S0 (2 Tc K V)
    and P U (2 Tc Tc V, P lower-triangular but multiplied whole) -- each
    product counted once, although the kernel runs three bf16 MMAs per product
    (hi.hi, hi.lo, lo.hi of the split fp32 operands)."""
    nchunks = (w.T + 63) // 64
    return w.N * w.HV * nchunks * (2 * 64 * w.K * w.V + 2 * 64 * 64 * w.V)


def time_prefill_state_stage(kda, reps, outs, stream, steps, stage=1):
    """µs per launch of one prefill stage (kda_prefill_stage; 1 = the state
    recurrence, the longest of the call's three kernels): CUDA events on the
    launching stream around eager launches that rotate over the replicas, each
    replica's workspace first filled by one whole call."""
    import torch

    fns = []
    with torch.cuda.stream(stream):
        for d, o in zip(reps, outs):
            ws = torch.empty(kda.prefill_workspace_bytes(d.N, d.T, d.HV, d.K, d.V), dtype=torch.uint8,
                             device=d.q.device)
            kda.kda_prefill(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, out=o, scale=d.scale, workspace=ws,
                            stream=stream)
            fns.append(lambda d=d, o=o, ws=ws: kda.kda_prefill(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx,
                                                               out=o, scale=d.scale, workspace=ws, stream=stream,
                                                               stage=stage))
        for f in fns[:3]:
            f()
    n = max(2 * len(fns), min(steps, 200))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        a.record(stream)
        for i in range(n):
            fns[i % len(fns)]()
        b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e3 / n, n


def measured_bf16_peak():
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure (a kernel
    timed on its own), else the recipe's earlier measurement on this machine."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.text = ""
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.cmd = ["nvidia-smi", "-i", gid, f"--query-gpu={','.join(self.FIELDS)}",
                        "--format=csv,noheader,nounits", "-lms", "100"]
        except Exception:
            self.cmd = None

    def __enter__(self):
        if self.cmd:
            try:
                self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                             text=True)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.text, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.text, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for rec in csv.reader(io.StringIO(self.text)):
            if len(rec) != len(self.FIELDS):
                continue
            try:
                rows.append([x.strip() for x in rec])
            except ValueError:
                continue
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm
def call_fn(kda, d, out, stream):
    if d.name.startswith("prefill_"):  # the chunked prefill over the workload's T tokens
        import torch

        ws = torch.empty(kda.prefill_workspace_bytes(d.N, d.T, d.HV, d.K, d.V), dtype=torch.uint8,
                         device=d.q.device)
        return lambda: kda.kda_prefill(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, out=out, scale=d.scale,
                                       workspace=ws, stream=stream)
    if d.packed or d.raw is not None or d.state_layout != "kv":  # the general entry point
        from linear_attention_recurrent_decode_b200 import workloads

        q, k, v = d.q, d.k, d.v
        if d.packed:
            _, (q, k, v) = workloads.pack_rows([d.q, d.k, d.v], pad=8)
        extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=d.eps) if d.gated else {}
        if d.raw is not None:
            r = d.raw
            extra.update(raw_gate=r.raw_gate, A_log=r.A_log, dt_bias=r.dt_bias, raw_beta=r.raw_beta)
        else:
            extra.update(g=d.g, beta=d.beta)
        return lambda: kda.kda_decode_ex(q, k, v, d.state, d.slot_idx, out=out, scale=d.scale,
                                         stream=stream, state_layout=d.state_layout, **extra)
    if d.gated:
        return lambda: kda.kda_decode_gated_rmsnorm(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx,
                                                    d.gate, d.norm_weight, eps=d.eps, out=out,
                                                    scale=d.scale, stream=stream)
    return lambda: kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, out=out,
                                  scale=d.scale, stream=stream)


def choose_replicas(touched_bytes: int, l2_bytes: int) -> int:
    """Enough replicas that the bytes touched between two uses of one replica
    exceed twice the L2 size."""
    return max(2, int(math.ceil(2 * l2_bytes / max(1, touched_bytes))) + 1)


def _oracle_gate(oracle, w):
    """(g, beta) for the oracle: as drawn, or activated from the serving form."""
    if w.raw is None:
        return w.g, w.beta
    r = w.raw
    return oracle.activate(r.raw_gate, r.A_log, r.dt_bias, r.raw_beta)


def time_cpu_oracle(w, budget_s: float = 8.0, max_calls: int = 200):
    """Median wall time of the fp64 oracle on the full call, all host cores."""
    import numpy as np

    import oracle

    threads = os.cpu_count() or 1
    pool = w.state_kv().double().numpy().copy()
    times = []
    t_end = time.perf_counter() + budget_s
    while len(times) < max_calls and (len(times) < 3 or time.perf_counter() < t_end):
        t0 = time.perf_counter()
        g, beta = _oracle_gate(oracle, w)
        oracle.kda_decode_ref(w.q, w.k, w.v, g, beta, None, w.slot_idx, w.scale,
                              gate=w.gate if w.gated else None,
                              norm_weight=w.norm_weight if w.gated else None, eps=w.eps,
                              threads=threads, state_inplace=pool)
        times.append(time.perf_counter() - t0)
    return statistics.median(times), threads, len(times)


class GraphRegion:
    """Exactly ``steps`` calls, rotating over the given callables (one per
    replica), timed on the device from CUDA graphs.

    Graphs: ``cycle`` (one call per replica, in order); the timed region (one
    graph of ``steps`` calls when that is at most ``SINGLE_GRAPH_MAX``, else
    ``cycle`` replayed steps // R times and a graph of the remainder); and
    ``tail``, the rest of the cycle after the remainder, replayed untimed after
    every region so that each region starts on replica 0 with every replica last
    touched R calls earlier (inputs larger than L2 stay cold).

    ``run`` enqueues, with no host synchronisation in between: a pre-roll of
    ``cycle`` replays lasting about ``preroll_s`` (so the clocks are at load and
    the first region starts on a busy stream, with no launch gap or idle GPU
    counted), then ``repeats`` regions, each between two CUDA events on the
    launching stream and followed by ``tail``.  Returns each region's
    milliseconds.  ``repeats`` = 0 picks an odd count (1..9) that keeps the
    regions to about a second in all."""

    SINGLE_GRAPH_MAX = 4096

    def __init__(self, calls, steps, stream, preroll_s, repeats):
        import torch

        self.stream = stream
        R = len(calls)
        rem = steps % R
        self.cycle = self._capture(calls)
        if steps <= self.SINGLE_GRAPH_MAX:
            self.timed = [self._capture([calls[i % R] for i in range(steps)])]
        else:
            self.timed = [self.cycle] * (steps // R) + ([self._capture(calls[:rem])] if rem else [])
        self.tail = self._capture(calls[rem:]) if rem else None
        # upload every graph (keeping the rotation: tail after each region), then
        # estimate the time of one cycle (all untimed)
        with torch.cuda.stream(stream):
            self.cycle.replay()
            for g in (self.timed[0], self.timed[-1]):
                g.replay()
                if self.tail:
                    self.tail.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(3):
                self.cycle.replay()
            b.record(stream)
        torch.cuda.synchronize()
        cycle_s = max(a.elapsed_time(b) / 3e3, 1e-6)
        self.preroll = max(2, int(math.ceil(preroll_s / cycle_s)))
        region_s = cycle_s * steps / R
        if repeats <= 0:
            repeats = max(1, min(9, int(1.0 / max(region_s, 1e-9))))
            repeats -= (repeats + 1) % 2  # odd: the median is one of the regions
        self.repeats = repeats

    def _capture(self, fns):
        import torch

        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(self.stream):
            with torch.cuda.graph(g, stream=self.stream):
                for fn in fns:
                    fn()
        return g

    def run(self):
        import torch

        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(self.repeats)]
        with torch.cuda.stream(self.stream):
            for _ in range(self.preroll):
                self.cycle.replay()
            for e0, e1 in ev:
                e0.record(self.stream)
                for g in self.timed:
                    g.replay()
                e1.record(self.stream)
                if self.tail:
                    self.tail.replay()
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    def release(self):
        self.cycle = self.timed = self.tail = None


def run_ours(args):
    import torch
    import torch.distributed as dist

    import linear_attention_recurrent_decode_b200 as kda
    from linear_attention_recurrent_decode_b200 import workloads

    rank, local_rank, world = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    kda.library()

    base = workloads.config(args.config, seed=rank_seed(0, rank))
    bytes_per_call = base.io_bytes() + 2 * base.state_bytes_touched()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = args.replicas or choose_replicas(base.state_bytes_touched() + base.io_bytes(), l2)
    reps = [base.to(dev)] + [workloads.config(args.config, seed=rank_seed(1 + r, rank)).to(dev)
                             for r in range(R - 1)]
    outs = [torch.empty(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16, device=dev) for w in reps]
    stream = torch.cuda.Stream(device=dev)
    calls = [call_fn(kda, d, o, stream) for d, o in zip(reps, outs)]

    # warm-up: W eager calls on the timing stream
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            calls[i % R]()
    torch.cuda.synchronize()

    timer = GraphRegion(calls, args.steps, stream, args.preroll_ms / 1e3, args.repeats)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if (rank == 0 and not args.no_clocks) else None
    if sampler:
        sampler.__enter__()
    t_wall0 = time.perf_counter()
    region_ms = timer.run()
    t_wall = time.perf_counter() - t_wall0
    if sampler:
        sampler.__exit__(None, None, None)
    if world > 1:
        dist.barrier()
    ms_rank = statistics.median(region_ms)
    ms_max = reduce_max(ms_rank, dev)
    timer.release()

    # the same calls launched one at a time from Python (no graph): what an
    # eager caller sees, host launch cost included
    n_eager = min(args.steps, 20_000)
    torch.cuda.synchronize()
    ea = torch.cuda.Event(enable_timing=True)
    eb = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(min(R, 8)):  # untimed lead-in: the first event is recorded on a busy stream
            calls[(n_eager + i) % R]()
        ea.record(stream)
        for i in range(n_eager):
            calls[i % R]()
        eb.record(stream)
    torch.cuda.synchronize()
    eager_us = reduce_max(ea.elapsed_time(eb), dev) * 1e3 / n_eager

    # prefill: the state recurrence alone (its roofline; see prefill_state_flops)
    stage = None
    if args.config.startswith("prefill_"):
        stage_us, stage_n = time_prefill_state_stage(kda, reps, outs, stream, args.steps)
        out_us, _ = time_prefill_state_stage(kda, reps, outs, stream, args.steps, stage=2)
        stage = (reduce_max(stage_us, dev), stage_n, reduce_max(out_us, dev))

    # end to end through the public API: pinned host inputs in, output back out
    n_e2e = min(args.steps, args.e2e_steps)
    if args.config.startswith("prefill_"):
        e2e = run_e2e_prefill(kda, base, dev, stream, n_e2e, world)
    else:
        e2e = run_e2e(kda, base, dev, stream, n_e2e, world, args.e2e_sets)
    floor = None if args.no_floor else copy_floor(base, dev, stream, R, args.steps, args.preroll_ms / 1e3)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    us_per_call_job = ms_max * 1e3 / (args.steps * world)
    launch_us = ms_max * 1e3 / args.steps
    peak, peak_kind = measured_peaks()
    achieved = bytes_per_call / (launch_us * 1e-6) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        t_cpu, cores, n_calls = time_cpu_oracle(base)
        cpu = {"value": t_cpu * 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n_calls} full calls of {args.config} (fp64 C loop, threads over (n,h))"}
    clocks = sampler.summary() if sampler else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                "algorithmic_bytes_per_launch": bytes_per_call,
                "traffic": profiled_traffic(args.config)}
    if stage is not None:
        # The prefill's longest kernel is its fp32 state recurrence on the CUDA
        # cores: flops against the fp32 ALU peak (the call's HBM view kept beside).
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        alu_peak = fp32_alu_peak_tflops(sms)
        flops = prefill_state_flops(base)
        tf = flops / (stage[0] * 1e-6) / 1e12
        roofline = {"bound": "alu", "kernel": "kda_prefill_state_kernel (stage 1: the state recurrence)",
                    "achieved": round(tf, 2), "peak": round(alu_peak, 1), "unit": "TFLOP/s",
                    "frac": round(tf / alu_peak, 4),
                    "peak_source": f"derived: {sms} SMs x 128 fp32 FMA lanes x 2 flop x 1965 MHz",
                    "algorithmic_flops_per_launch": flops, "launch_us": round(stage[0], 2),
                    "launches_timed": stage[1], "traffic": None,
                    "call_hbm": {"achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                                 "frac": round(achieved / peak, 4), "algorithmic_bytes_per_call": bytes_per_call}}
        bf16_peak, bf16_kind = measured_bf16_peak()
        oflops = prefill_output_flops(base)
        otf = oflops / (stage[2] * 1e-6) / 1e12
        roofline["tensor_kernel"] = {
            "kernel": "kda_prefill_output_kernel (stage 2: chunk outputs, tcgen05 bf16 MMAs)",
            "bound": "tensor", "achieved": round(otf, 2), "peak": bf16_peak, "unit": "TFLOP/s",
            "frac": round(otf / bf16_peak, 4), "peak_source": bf16_kind, "algorithmic_flops_per_launch": oflops,
            "launch_us": round(stage[2], 2),
            "note": "each fp32 product counted once; the kernel issues three bf16 MMAs per product"}
    line = {
        "metric": METRIC, "value": round(us_per_call_job, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; bf16 q/k/v, fp32 g/beta/state)",
        "config": {"workload": args.config, "N": base.N, "T": base.T, "HV": base.HV, "K": base.K,
                   "V": base.V, "num_slots": base.num_slots, "gated": base.gated,
                   "replicas": R, "l2": f"inputs larger than L2: {R} rotating replicas touch "
                   f"{R * (base.state_bytes_touched() + base.io_bytes()) / 1e6:.0f} MB > 2 x "
                   f"{l2 / 1e6:.0f} MB L2",
                   "timing": f"CUDA graph replay, CUDA events on the launching stream: {timer.repeats} "
                             f"regions of exactly {args.steps} calls behind a {timer.preroll}-replay "
                             "untimed pre-roll, no host sync in between; value from the median region",
                   "region_us_per_call": [round(x * 1e3 / args.steps, 4) for x in region_ms],
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "gbs": round(achieved, 1),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "eager": {"value": round(eager_us, 3), "unit": UNIT, "steps": n_eager,
                  "how": "the same calls on the same rotating replicas, launched one at a time from "
                         "Python (no CUDA graph)"},
        "clocks": clocks,
        "floor": floor,
        "gpu_launches": args.steps * (3 if args.config.startswith("prefill_") else 1),
        "wall_s_timed": round(t_wall, 3),
    }
    print(json.dumps(line), flush=True)


def _packed(tensors: dict, alloc):
    """One buffer holding every tensor of ``tensors`` (16-byte aligned slices),
    plus views of it with the tensors' shapes and dtypes."""
    import torch

    offs, off = {}, 0
    for k, t in tensors.items():
        offs[k] = off
        off += (t.numel() * t.element_size() + 15) // 16 * 16
    buf = alloc(off)
    views = {k: buf[offs[k]:offs[k] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for k, t in tensors.items()}
    return buf, views


def copy_floor(w, dev, stream, R, steps, preroll_s):
    """Per-call time of a plain in-place elementwise op (torch's x.mul_(c)) over
    exactly the state bytes one decode call reads and writes, with the same
    rotation over R buffers and the same graph-replay timing as the decode: the
    practical floor for moving those bytes once each way per call on this GPU."""
    import torch

    n = w.state_bytes_touched() // 4
    bufs = [torch.randn(n, device=dev) for _ in range(R)]
    fns = [(lambda b=b: b.mul_(1.0001)) for b in bufs]
    timer = GraphRegion(fns, steps, stream, preroll_s, repeats=0)
    torch.cuda.synchronize()
    ms = statistics.median(timer.run())
    timer.release()
    us = ms * 1e3 / steps
    return {"what": "torch in-place x.mul_(c) over the same state bytes (read + write), same replica "
                    "rotation and graph-replay timing", "us_per_call": round(us, 3),
            "bytes_per_call": 2 * n * 4, "gbs": round(2 * n * 4 / (us * 1e-6) / 1e9, 1)}


def _host_step(kda, w, dev, stream, pool):
    """One staging set: the step's inputs packed in one pinned host buffer (as a
    serving host would stage them), its device copy, and a HostStep bound to
    them and to ``pool``."""
    import torch

    inputs = {k: t for k, t in w.tensors().items() if k != "state"}
    host_buf, host = _packed(inputs, lambda n: torch.empty(n, dtype=torch.uint8).pin_memory())
    for k, t in inputs.items():
        host[k].copy_(t)
    dev_buf, devv = _packed(inputs, lambda n: torch.empty(n, dtype=torch.uint8, device=dev))
    out_d = torch.empty(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16, device=dev)
    out_h = torch.empty(out_d.shape, dtype=torch.bfloat16).pin_memory()
    extra = dict(gate=devv["gate"], norm_weight=devv["norm_weight"], eps=w.eps) if w.gated else {}
    if w.raw is not None:
        extra.update(raw_gate=devv["raw_gate"], A_log=devv["A_log"], dt_bias=devv["dt_bias"],
                     raw_beta=devv["raw_beta"])
    else:
        extra.update(g=devv["g"], beta=devv["beta"])
    step = kda.HostStep(devv["q"], devv["k"], devv["v"], pool, devv["slot_idx"], host_in=host_buf,
                        dev_in=dev_buf, host_out=out_h, out=out_d, stream=stream, scale=w.scale,
                        state_layout=w.state_layout, **extra)
    return step, host_buf, dev_buf, out_h


def _timed_steps(fn, steps, stream, lead_in, copy_stream=None):
    """Device time of ``steps`` calls of fn between events on ``stream``, after
    ``lead_in`` untimed calls enqueued without a host sync (the first event is
    recorded on a busy stream); a copy stream waits for the first event, so no
    copy of the timed steps starts before it."""
    import torch

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(lead_in):
            fn()
        e0.record(stream)
        if copy_stream is not None:
            copy_stream.wait_event(e0)
        for _ in range(steps):
            fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_e2e(kda, w, dev, stream, steps, world, nsets=2):
    """µs per step with each step's inputs copied from pinned host memory and
    its output copied back, through the public API; the state pool stays
    resident on the GPU.  The value is the pipelined form (``HostPipeline``,
    the C ABI's ``kda_decode_host_pipelined``): ``nsets`` staging sets used in
    turn, each step's copy in on a second stream so that it overlaps the
    previous steps' kernels and copies out.  Also reported: the same steps one
    after another on one stream (``HostStep``, ``kda_decode_host``), and the
    copy in alone."""
    import torch

    pool = w.state.to(dev)
    copy_stream = torch.cuda.Stream(device=dev)
    sets = [_host_step(kda, w, dev, stream, pool) for _ in range(nsets)]
    pipe = kda.HostPipeline([s[0] for s in sets], copy_stream)
    h2d = sets[0][1].numel()  # the packed buffer each step copies (inputs and their 16-byte alignment)
    d2h = sets[0][3].numel() * sets[0][3].element_size()

    for _ in range(10):
        pipe()
    torch.cuda.synchronize()
    ms_eager = reduce_max(_timed_steps(pipe, steps, stream, lead_in=4, copy_stream=copy_stream), dev)
    # The same calls captured once into a CUDA graph (as a serving loop replays
    # its decode steps): each replay runs `per_graph` steps, copies included.
    per_graph = nsets * max(1, min(steps, 64) // nsets)
    reps = max(1, -(-steps // per_graph))
    graph_note = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            copy_stream.wait_stream(stream)  # fork the copy stream into the capture
            pipe.rearm()
            for _ in range(per_graph):
                pipe()
            stream.wait_stream(copy_stream)  # and join it back
        torch.cuda.synchronize()
        ms_graph = _timed_steps(graph.replay, reps, stream, lead_in=2)
        del graph
    except RuntimeError as exc:  # report the eager pipelined figure instead, and why
        torch.cuda.synchronize()
        graph_note = f"graph capture failed ({str(exc).splitlines()[0][:120]}); value is the eager pipelined figure"
        ms_graph = ms_eager * reps * per_graph / steps
    ms_graph = reduce_max(ms_graph, dev)
    serial = sets[0][0]
    ms_serial = reduce_max(_timed_steps(serial, steps, stream, lead_in=4), dev)
    host_buf, dev_buf = sets[0][1], sets[0][2]
    ms_copy = reduce_max(_timed_steps(lambda: dev_buf.copy_(host_buf, non_blocking=True), steps, stream,
                                      lead_in=4), dev)
    return {"value": round(ms_eager * 1e3 / (steps * world), 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "graph_us": round(ms_graph * 1e3 / (reps * per_graph * world), 3),
            "serial_us": round(ms_serial * 1e3 / (steps * world), 3),
            "h2d_copy_us": round(ms_copy * 1e3 / steps, 3),
            "how": "kda_decode_host_pipelined through HostPipeline, one call per step from Python: the copy of "
                   "the step's packed inputs from pinned host memory (on a copy stream, overlapping the previous "
                   f"step), the decode kernel and the copy of the output back to pinned host memory; {nsets} staging "
                   "sets in turn; the state pool stays resident on the GPU.  graph_us: the same calls captured "
                   f"{per_graph} at a time in a CUDA graph and replayed; serial_us: copy in, kernel and copy out "
                   "one after another on one stream (kda_decode_host); h2d_copy_us: the copy in alone",
            **({"note": graph_note} if graph_note else {})}


def run_e2e_prefill(kda, w, dev, stream, steps, world):
    """µs per prefill call with the call's inputs copied from pinned host memory
    (one copy per input tensor) and its output copied back, through the public
    Python API; the state pool and the workspace stay on the device."""
    import torch

    inputs = {k: t for k, t in w.tensors().items() if k != "state"}
    host = {k: t.pin_memory() for k, t in inputs.items()}
    devv = {k: torch.empty_like(t, device=dev) for k, t in inputs.items()}
    pool = w.state.to(dev)
    out_d = torch.empty(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16, device=dev)
    out_h = torch.empty(out_d.shape, dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(kda.prefill_workspace_bytes(w.N, w.T, w.HV, w.K, w.V), dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()

    def step():
        for k, t in host.items():
            devv[k].copy_(t, non_blocking=True)
        kda.kda_prefill(devv["q"], devv["k"], devv["v"], devv["g"], devv["beta"], pool, devv["slot_idx"],
                        out=out_d, scale=w.scale, workspace=ws, stream=stream)
        out_h.copy_(out_d, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        step()  # untimed lead-in: the first event is recorded on a busy stream
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1), dev)
    return {"value": round(ms * 1e3 / (steps * world), 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "how": "per step: copies of the inputs from pinned host memory, kda_prefill, copy of the output back "
                   "(torch copies around the library call); state pool and workspace resident on the GPU"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """fp64 oracle on the host cores, same workload/metric; rank 0 only."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    from linear_attention_recurrent_decode_b200 import workloads
    import oracle

    w = workloads.config(args.config)
    units = w.N * w.HV
    threads = os.cpu_count() or 1
    pool = w.state_kv().double().numpy().copy()
    kw = dict(gate=w.gate, norm_weight=w.norm_weight, eps=w.eps) if w.gated else dict(eps=w.eps)

    g, beta = _oracle_gate(oracle, w)  # the serving form's activation, once

    def one(lo, hi, thr):
        t0 = time.perf_counter()
        oracle.kda_decode_ref(w.q, w.k, w.v, g, beta, None, w.slot_idx, w.scale, threads=thr,
                              units=(lo, hi), state_inplace=pool, **kw)
        return time.perf_counter() - t0

    t_full = min(one(0, units, threads) for _ in range(2))
    budget = args.reference_budget_s
    total = args.steps + args.warmup
    if total * t_full <= budget:
        per_step, thr = units, threads
    else:
        # Bounded samples: single-threaded (no per-call thread start-up), as
        # many (n, h) units per step as the budget allows given the measured
        # fixed cost of a call and cost of a unit.
        t1 = min(one(0, 1, 1) for _ in range(3))
        t8 = min(one(0, min(8, units), 1) for _ in range(3))
        t_unit = max((t8 - t1) / max(1, min(8, units) - 1), 1e-7)
        overhead = max(t1 - t_unit, 0.0)
        per_step = int(max(1, min(units, (budget / total - overhead) / t_unit)))
        thr = 1
    times = []
    lo = 0
    for i in range(total):
        hi = min(units, lo + per_step)
        dt = one(lo, hi, thr)
        if i >= args.warmup:
            times.append(dt * units / (hi - lo))
        lo = 0 if hi >= units else hi
    us = statistics.mean(times) * 1e6
    sample = (f"each step: {per_step} of the {units} (n,h) units of {args.config}, single-threaded, "
              f"scaled to a full call (the run is bounded to about {budget:.0f} s)"
              if per_step < units else f"each step: one full call of {args.config}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; bf16 q/k/v, fp32 g/beta/state)",
        "config": {"workload": args.config, "N": w.N, "T": w.T, "HV": w.HV, "K": w.K, "V": w.V,
                   "num_slots": w.num_slots, "gated": w.gated},
        "cpu_baseline": {"value": round(us, 3), "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(us, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200_000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--config", default="n32_t1_hv8")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--replicas", type=int, default=0, help="0 = enough to exceed 2x L2")
    ap.add_argument("--e2e-steps", type=int, default=5000)
    ap.add_argument("--e2e-sets", type=int, default=2,
                    help="staging sets the pipelined end-to-end steps use in turn (>= 1)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-floor", action="store_true", help="skip the in-place copy-floor reference")
    ap.add_argument("--reference-budget-s", type=float, default=90.0)
    ap.add_argument("--preroll-ms", type=float, default=300.0,
                    help="untimed graph replays enqueued ahead of the timed regions")
    ap.add_argument("--repeats", type=int, default=0,
                    help="timed regions of --steps calls (0 = an odd count filling about a second)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps < 1:
        raise SystemExit("--steps must be >= 1")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
