#!/usr/bin/env python
"""Benchmark of the KDA layer-half decode step (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload b8|b1|b12|b64]

A step is one kda_decode_step: one token for every sequence of the batch
through projections, gates, the in-place state update, readout and output
projection.  The default workload is batch 8, hidden 4096, 32 heads of
128 x 128.  Each rank runs its own independent batch (data parallel over
sequences, no collective on the data path); ``value`` is the whole-job
decode steps/s, the max step time over ranks.

Timing: W warm-up steps, then exactly K steps between CUDA events on the
library's stream, bracketed by a barrier and a device synchronize.  Steps
rotate over enough copies of weights + state (+ x, out) to exceed twice the
L2 size, so every step streams from HBM, including the write-back of the
previous step's state.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_layer_kda_b200 import inputs as I  # noqa: E402

METRIC = "KDA layer-half decode steps/s & tokens/s at batch 8; achieved HBM GB/s vs 8 TB/s"
WORKLOADS = {"b8": 1, "b1": 2, "b12": 3, "b64": 4}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def ideal_bytes(s: I.KdaShape, B: int, out_bytes: int = 4) -> int:
    """Algorithmic bytes of one step: weights, scales, gate weights, state read + write, x, out."""
    H, Dk, Dv, nh, r = s.hidden, s.dk_total, s.dv_total, s.num_heads, s.alpha_rank
    fp8 = 2 * Dk * H + Dv * H + H * Dv
    scales = 4 * ((Dk // 128) * (H // 128) * 2 + (Dv // 128) * (H // 128) + (H // 128) * (Dv // 128))
    gates = 2 * (r * H + Dk * r + nh * H)
    state = 2 * B * nh * s.head_dk * s.head_dv * 4
    return fp8 + scales + gates + state + B * H * 2 + B * H * out_bytes


def ideal_flops(s: I.KdaShape, B: int) -> int:
    H, Dk, Dv, nh, r = s.hidden, s.dk_total, s.dv_total, s.num_heads, s.alpha_rank
    proj = 2 * B * (2 * Dk * H + Dv * H + H * Dv + r * H + Dk * r + nh * H)
    return proj + 8 * B * nh * s.head_dk * s.head_dv


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while it runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, path: str):
        self.path = path
        self.proc = None
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, n = [], [], set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in open(self.path):
            c = [x.strip() for x in ln.split(",")]
            if len(c) < 9:
                continue
            try:
                sm.append(float(c[1]))
                smax.append(float(c[2]))
            except ValueError:
                continue
            n += 1
            for nm, v in zip(names, c[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": n}


def gpu_id_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------------ CPU baseline (oracle)

def oracle_rate(shape: I.KdaShape, inp, seqs: int, budget_s: float, max_steps: int):
    """Oracle decode steps over `seqs` sequences; returns (full-batch steps/s, steps run, cores)."""
    import oracle
    m = oracle.OracleModel(inp, batch=seqs)
    S = inp.state0[:seqs].astype(np.float64).copy()
    n, t0 = 0, time.perf_counter()
    while n < max_steps:
        m.step(inp.x[0][:seqs], S)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    m.close()
    return (n * seqs / shape.batch) / dt, n, oracle.num_threads()


def run_reference(args, shape, rank):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    inp = I.generate(shape.replace(steps=1))
    seqs = shape.batch if args.steps <= 50 else 1
    m = oracle.OracleModel(inp, batch=seqs)
    S = inp.state0[:seqs].astype(np.float64).copy()
    for _ in range(args.warmup):
        m.step(inp.x[0][:seqs], S)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        m.step(inp.x[0][:seqs], S)
    dt = time.perf_counter() - t0
    m.close()
    full_steps_per_s = (args.steps * seqs / shape.batch) / dt
    sample = (f"each step: one fp64 oracle decode step over {seqs} of the {shape.batch} sequences "
              f"(rank-1 form, OpenMP), scaled to full-batch steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": full_steps_per_s, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / full_steps_per_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, args.gpus, "cpu"),
        "cpu_baseline": {"value": full_steps_per_s, "unit": "steps/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": full_steps_per_s, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rank_inputs(shape: I.KdaShape, rank: int, world: int):
    """Inputs of one rank: weights shared by all ranks; x and state are this rank's own
    sequences, rows rank*B .. rank*B + B - 1 of the job's counter-based streams, so the N
    ranks together hold exactly the sequences of one batch of N*B (data parallel, no
    collective on the data path)."""
    inp = I.generate(shape.replace(steps=1))
    if world > 1:
        B = shape.batch
        inp.x[0] = I.gen_x(shape, 0, batch=B, row0=rank * B)
        inp.state0 = I.gen_state(shape, batch=B, row0=rank * B)
    return inp


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_steps_per_s(ms_per_step_slowest: float, world: int) -> float:
    """Whole-job decode steps/s: every rank advances its own batch once per step."""
    return world * 1000.0 / ms_per_step_slowest


def workload_config(shape, n, l2_note):
    return {"workload": shape.name, "batch_per_gpu": shape.batch, "global_batch": shape.batch * n,
            "hidden": shape.hidden, "num_heads": shape.num_heads, "head_dk": shape.head_dk,
            "head_dv": shape.head_dv, "alpha_rank": shape.alpha_rank,
            "weights": "FP8 E4M3 q/k/v/o with fp32 128x128 block scales; bf16 alpha (low rank) and beta",
            "state": "fp32 [B, nh, dk, dv], updated in place", "out": "fp32",
            "parallelism": f"dp{n} (independent sequences per GPU, weights replicated, no collective)",
            "l2": l2_note}


# ------------------------------------------------------------------ our arm

def run_ours(args, shape, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from linear_attention_layer_kda_b200 import binding, tensors

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    B = shape.batch
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))

    inp = rank_inputs(shape, rank, world)
    set_bytes = ideal_bytes(shape, B)
    R = max(2, math.ceil(2 * l2 / set_bytes))
    wts = [tensors.to_device_weights(inp, dev) for _ in range(R)]
    ws = [tensors.weights_struct(w) for w in wts]
    states = [tensors.state_tensor(inp.state0, dev) for _ in range(R)]
    xs = [tensors.bf16_tensor(inp.x[0], dev) for _ in range(R)]
    outs = [torch.empty(B, shape.hidden, device=dev, dtype=torch.float32) for _ in range(R)]
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B,
                             engine=args.engine)
    engine = dec.engine(B)
    launches = dec.launches_per_step(B)

    def one(i):
        j = i % R
        dec.step(xs[j], ws[j], states[j], outs[j])

    for i in range(max(3, args.warmup)):
        one(i)
    dec.sync()
    torch.cuda.synchronize()

    clk = ClockSampler(gpu_id_for(local_rank), os.path.join(args.outdir, f"clocks_rank{rank}.csv")) \
        if rank == 0 else None
    # untimed load window so the clock sampler sees the step loop for about a second
    t_end = time.perf_counter() + (args.clock_window if clk else 0.0)
    i = 0
    while time.perf_counter() < t_end:
        one(i)
        i += 1
        if i % 256 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        one(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    dec.sync()  # raises on a recorded device-side timeout
    if world > 1:
        dist.barrier()
    ms_total = ev0.elapsed_time(ev1)
    clocks = clk.stop() if clk else None

    ms_total = max_over_ranks(ms_total, world, dev)
    ms_per_step = ms_total / args.steps
    value = job_steps_per_s(ms_per_step, world)

    # end to end through the host-buffer entry point: H2D x, step, D2H out, sync, every step,
    # on every rank; the slowest rank's wall time sets the job's rate
    xh = torch.from_numpy(inp.x[0].view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty(B, shape.hidden, dtype=torch.float32).pin_memory()
    n_e2e = args.e2e_steps if args.e2e_steps > 0 else max(10, min(args.steps, 2000))
    for i in range(3):
        dec.step_host(xh, ws[i % R], states[i % R], oh)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(n_e2e):
        dec.step_host(xh, ws[i % R], states[i % R], oh)
    dt = max_over_ranks(time.perf_counter() - t0, world, dev)
    e2e = {"value": job_steps_per_s(1000.0 * dt / n_e2e, world), "unit": "steps/s",
           "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(oh.numel() * 4), "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, cores = oracle_rate(shape, inp, seqs=B, budget_s=args.cpu_seconds, max_steps=1000)
        cpu = {"value": rate, "unit": "steps/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} fp64 oracle decode steps of the same workload (batch {B}, rank-1 form, "
                         f"OpenMP), about {args.cpu_seconds:.0f} s of CPU work"}

    dec.close()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = measured_peaks()
    hbm_peak = peaks.get("hbm_gbs")
    peak_src = "measured" if hbm_peak else "fallback"
    hbm_peak = float(hbm_peak or FALLBACK_HBM_GBS)
    ib = ideal_bytes(shape, B)
    achieved = ib / (ms_per_step * 1e-3) / 1e9
    traffic = None
    tfile = os.path.join(ROOT, "profiles", f"traffic_{shape.name}.json")
    if os.path.exists(tfile):
        try:
            tj = json.load(open(tfile))
            if tj.get("engine") == engine and tj.get("kernel_rev") == kernel_rev():
                traffic = tj.get("dram_bytes_per_launch")
        except (OSError, ValueError):
            traffic = None
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(shape, world, f"rotating {R} weight+state sets of {set_bytes / 1e6:.1f} MB "
                                               f"(> 2x the {l2 / 2 ** 20:.0f} MiB L2)"),
        "tokens_per_s": value * B,
        "hbm_gbs": achieved, "hbm_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "engine": {1: "simple", 2: "fused"}.get(engine, str(engine)),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": ("whole step (one persistent kernel)" if launches == 1 else
                                f"whole step ({launches} kernels)"),
                     "algorithmic_bytes_per_launch": ib if launches == 1 else None,
                     "algorithmic_bytes_per_step": ib},
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "cpu_baseline": cpu,
        "ideal_flops_per_step": ideal_flops(shape, B),
    }
    print(json.dumps(line), flush=True)
    return 0


def kernel_rev() -> str:
    """Hash of the CUDA sources: a stored ncu traffic figure is reported only for the kernel it measured."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_attention_layer_kda_b200", "csrc")
    for n in ("common.cuh", "sm100.cuh", "fused.cuh", "fused.cu", "schedule.cu", "simple.cu"):  # the engines
        for line in open(os.path.join(d, n)):
            code = line.split("//", 1)[0].strip()  # comments and layout do not change the kernel
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default="b8")
    ap.add_argument("--engine", type=int, default=0, help="0 auto, 1 simple, 2 fused")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-window", type=float, default=1.0,
                    help="seconds of untimed steps while nvidia-smi samples clocks before the timed region")
    ap.add_argument("--e2e-steps", type=int, default=0, help="steps of the host-buffer end-to-end loop")
    ap.add_argument("--outdir", default=os.path.join(ROOT, "bench_out"), help="where the clock samples go")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    os.makedirs(args.outdir, exist_ok=True)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    shape = I.CONFIGS[WORKLOADS[args.workload]]
    if args.impl == "reference":
        return run_reference(args, shape, rank)
    return run_ours(args, shape, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
