#!/usr/bin/env python
"""Benchmark of the KDA layer-half decode step (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload b8|b1|b12|b64]

With --gpus N > 1 and no torchrun environment, the script starts N ranks of
itself under torch.distributed.run (one process per GPU) and returns their
exit status.

A step is one kda_decode_step: one token for every sequence of the batch
through projections, gates, the in-place state update, readout and output
projection.  The default workload is batch 8, hidden 4096, 32 heads of
128 x 128.  Each rank runs its own independent batch (data parallel over
sequences, no collective on the data path); ``value`` is the whole-job
decode steps/s, the max step time over ranks.

Timing: W warm-up steps, then exactly K steps between CUDA events on the
library's stream, bracketed by a barrier and a device synchronize; an event
after every step gives the median, p10 and p90 of the per-step times.  Steps
rotate over enough copies of weights + state (+ x, out) to exceed twice the
L2 size, so every step streams from HBM, including the write-back of the
previous step's state.  SM clocks and clock-event reasons are sampled through
NVML while the timed steps run.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import socket
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_layer_kda_b200 import inputs as I  # noqa: E402

METRIC = "KDA layer-half decode steps/s & tokens/s at batch 8; achieved HBM GB/s vs 8 TB/s"
WORKLOADS = {"b8": 1, "b1": 2, "b12": 3, "b64": 4}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def prefill_flops(s: I.KdaShape, rows: int) -> int:
    """Multiply-adds x 2 of a prefill's projections for `rows` token rows."""
    H, Dk, Dv, nh, r = s.hidden, s.dk_total, s.dv_total, s.num_heads, s.alpha_rank
    return 2 * rows * (2 * Dk * H + Dv * H + H * Dv + nh * H + r * H + Dk * r)


def ideal_bytes(s: I.KdaShape, B: int, out_bytes: int = 4, tokens: int = 1) -> int:
    """Algorithmic bytes of one step: weights, scales, gate weights, state read + write, x, out
    (x and out for every token of every sequence; the state is read and written once)."""
    H, Dk, Dv, nh, r = s.hidden, s.dk_total, s.dv_total, s.num_heads, s.alpha_rank
    fp8 = 2 * Dk * H + Dv * H + H * Dv
    scales = 4 * ((Dk // 128) * (H // 128) * 2 + (Dv // 128) * (H // 128) + (H // 128) * (Dv // 128))
    gates = 2 * (r * H + Dk * r + nh * H)
    state = 2 * B * nh * s.head_dk * s.head_dv * 4
    return fp8 + scales + gates + state + B * tokens * H * (2 + out_bytes)


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
    """NVML sampling of the SM clock, power and clock-event reasons of one GPU.

    A background thread samples about every `period` seconds; `mark()` takes one
    sample at once (called right after the timed steps are enqueued, while the GPU
    runs them).  `stop(t0, t1)` reports the samples taken inside [t0, t1], the
    host-clock span of the timed region; if none fell inside (a timed region far
    shorter than the period), the marked sample and the samples next to the
    window stand for it and `in_window` says so."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_uuid: str, period: float = 0.002):
        self.samples = []  # (host time, sm MHz, max sm MHz, power W, reasons mask)
        self.err = None
        self.period = period
        self._stop = threading.Event()
        self._lock = threading.Lock()
        try:
            import pynvml as nv
            nv.nvmlInit()
            u = device_uuid if device_uuid.startswith("GPU-") else "GPU-" + device_uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(u)
            self.nv = nv
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
        except Exception as e:  # noqa: BLE001 - no NVML: report why, time anyway
            self.nv = None
            self.err = f"nvml unavailable: {e}"
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _sample(self):
        nv = self.nv
        t = time.perf_counter()
        sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        except Exception:  # noqa: BLE001
            pw = None
        rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        with self._lock:
            self.samples.append((t, sm, self.max_mhz, pw, rs))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(self.period)

    def mark(self):
        if self.nv is not None:
            try:
                self._sample()
            except Exception as e:  # noqa: BLE001
                self.err = str(e)

    def stop(self, t0: float, t1: float) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err], "samples": 0, "in_window": 0}
        self._stop.set()
        self.thread.join(timeout=5)
        with self._lock:
            allv = sorted(self.samples)
        inside = [v for v in allv if t0 <= v[0] <= t1]
        use = inside
        if not use:  # nearest samples on both sides of a very short window
            before = [v for v in allv if v[0] < t0][-1:]
            after = [v for v in allv if v[0] > t1][:1]
            use = before + after
        reasons = set()
        for v in use:
            for name, attr in self.REASONS:
                if v[4] & int(getattr(self.nv, attr, 0)):
                    reasons.add(name)
        pw = [v[3] for v in use if v[3] is not None]
        return {"sm_mhz": statistics.median(v[1] for v in use) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "power_w_max": max(pw) if pw else None, "samples": len(use), "in_window": len(inside),
                "source": "nvml, sampled while the timed steps ran"}


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# ------------------------------------------------------------------ CPU baseline (oracle)

def oracle_rate(shape: I.KdaShape, inp, seqs: int, budget_s: float, max_steps: int, threads: int = 0):
    """Oracle decode steps over `seqs` sequences; returns (full-batch steps/s, steps run, threads used).

    threads = 0 keeps OpenMP's default (every host core)."""
    import oracle
    if threads:
        oracle.set_num_threads(threads)
    m = oracle.OracleModel(inp, batch=seqs)
    S = inp.state0[:seqs].astype(np.float64).copy()
    n, t0 = 0, time.perf_counter()
    try:
        while n < max_steps:
            m.step(inp.x[n % len(inp.x)][:seqs], S)
            n += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        used = oracle.num_threads()
    finally:
        m.close()
        if threads:
            oracle.set_num_threads(os.cpu_count() or 1)
    return (n * seqs / shape.batch) / dt, n, used


L2_ASSUMED = 126 * 2 ** 20  # B200 L2; the GPU arm uses the device's own figure if it is larger


def rotation_sets(shape: I.KdaShape, l2: int = L2_ASSUMED) -> int:
    """Copies of (weights, state, x, out) the steps rotate over so that the set exceeds twice L2."""
    return max(2, math.ceil(2 * l2 / ideal_bytes(shape, shape.batch)))


def workload_config(shape, n, sets):
    """The workload as both arms report it (identical dictionaries for the same shape and N)."""
    steps_note = (f"{shape.steps} sequential decode steps, fresh x each step, state carried in place"
                  if shape.steps > 1 else "one decode step per timed iteration")
    return {"workload": shape.name, "batch_per_gpu": shape.batch, "global_batch": shape.batch * n,
            "hidden": shape.hidden, "num_heads": shape.num_heads, "head_dk": shape.head_dk,
            "head_dv": shape.head_dv, "alpha_rank": shape.alpha_rank,
            "weights": "FP8 E4M3 q/k/v/o with fp32 128x128 block scales; bf16 alpha (low rank) and beta",
            "state": "fp32 [B, nh, dk, dv], updated in place", "out": "fp32", "steps": steps_note,
            "parallelism": f"dp{n} (independent sequences per GPU, weights replicated, no collective)",
            "l2": f"inputs larger than L2: steps rotate over {sets} copies of weights + state "
                  f"({ideal_bytes(shape, shape.batch) / 1e6:.1f} MB each, > 2x the L2)"}


def run_reference(args, shape, rank, world):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only; other ranks exit at once)."""
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    steps = max(1, shape.steps)
    inp = I.generate(shape.replace(steps=steps))
    seqs = shape.batch if args.steps <= 50 else 1
    m = oracle.OracleModel(inp, batch=seqs)
    S = inp.state0[:seqs].astype(np.float64).copy()
    for i in range(args.warmup):
        m.step(inp.x[i % steps][:seqs], S)
    t0 = time.perf_counter()
    for i in range(args.steps):
        m.step(inp.x[i % steps][:seqs], S)
    dt = time.perf_counter() - t0
    m.close()
    full_steps_per_s = (args.steps * seqs / shape.batch) / dt
    sample = (f"each step: one fp64 oracle decode step over {seqs} of the {shape.batch} sequences "
              f"(rank-1 form, OpenMP), scaled to full-batch steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": full_steps_per_s, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / full_steps_per_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, world, rotation_sets(shape)),
        "cpu_baseline": {"value": full_steps_per_s, "unit": "steps/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": full_steps_per_s, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def token_rows(xs, T):
    """x of T consecutive tokens of every sequence as one [B * T, H] array (row b * T + t)."""
    return np.ascontiguousarray(np.stack(xs[:T], axis=1).reshape(-1, xs[0].shape[1]))


def rank_inputs(shape: I.KdaShape, rank: int, world: int):
    """Inputs of one rank: weights shared by all ranks; x and state are this rank's own
    sequences, rows rank*B .. rank*B + B - 1 of the job's counter-based streams, so the N
    ranks together hold exactly the sequences of one batch of N*B (data parallel, no
    collective on the data path)."""
    steps = max(1, shape.steps)
    inp = I.generate(shape.replace(steps=steps))
    if world > 1:
        B = shape.batch
        for t in range(steps):
            inp.x[t] = I.gen_x(shape, t, batch=B, row0=rank * B)
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


def job_steps_per_s(ms_per_step_slowest: float, world: int, tp: bool = False) -> float:
    """Whole-job decode steps/s: every rank advances its own batch once per step (data
    parallel), or all ranks advance one batch together (tensor parallel by heads)."""
    return (1 if tp else world) * 1000.0 / ms_per_step_slowest


def step_percentiles(step_ms):
    """median, p10, p90 of per-step times (ms)."""
    v = np.asarray(step_ms, dtype=np.float64)
    return float(np.median(v)), float(np.percentile(v, 10)), float(np.percentile(v, 90))


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
    l2 = max(L2_ASSUMED, int(getattr(props, "L2_cache_size", L2_ASSUMED)))

    TK = args.tokens if args.prefill <= 0 else args.prefill
    if TK > 1:
        shape = shape.replace(steps=max(shape.steps, TK))
    full_shape = shape
    if args.tp:  # this rank's heads: their weights and state, x and W_a_down whole
        from linear_attention_layer_kda_b200 import tp
        inp = tp.shard_inputs(I.generate(shape.replace(steps=max(1, shape.steps))), rank, world)
        shape = inp.shape
    else:
        inp = rank_inputs(shape, rank, world)
    T = len(inp.x)  # fresh x per step for multi-step workloads
    set_bytes = ideal_bytes(shape, B, tokens=TK)
    R = rotation_sets(shape, l2)
    wts = [tensors.to_device_weights(inp, dev) for _ in range(R)]
    ws = [tensors.weights_struct(w) for w in wts]
    states = [tensors.state_tensor(inp.state0, dev) for _ in range(R)]
    if TK > 1:  # one multi-token step: x of T consecutive tokens of every sequence
        xs = [tensors.bf16_tensor(token_rows(inp.x, TK), dev)]
        T = 1
    else:
        xs = [tensors.bf16_tensor(inp.x[t], dev) for t in range(T)]
    outs = [torch.empty(B * TK, shape.hidden, device=dev, dtype=torch.float32) for _ in range(R)]
    prefill = args.prefill > 0
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank,
                             B if prefill else B * TK, engine=args.engine)
    if args.tp:  # the out sum over ranks inside the fused kernel, over peer memory
        from linear_attention_layer_kda_b200 import tp
        tp.exchange_handles(dec, rank, world)
    if prefill:
        # this library's kernels per call (weight and activation splits, the chunk preparation and
        # scan) and the cuBLASLt GEMMs of the projections, beside them
        engine, launches, lib_launches = "prefill", 8, 13  # fp32 out
    else:
        engine = dec.engine(B) if TK == 1 else dec.tokens_engine(B, TK)
        launches = dec.launches_per_step(B) if TK == 1 else (1 if engine == 2 else dec.launches_per_step(B))
        lib_launches = 0

    def one(i):
        j = i % R
        if prefill:
            dec.prefill(xs[0], ws[j], states[j], outs[j], B, TK, args.chunk)
        elif TK == 1:
            dec.step(xs[i % T], ws[j], states[j], outs[j])
        else:
            dec.step_tokens(xs[0], ws[j], states[j], outs[j], B, TK)

    for i in range(max(3, args.warmup)):
        one(i)
    dec.sync()
    torch.cuda.synchronize()

    clk = ClockSampler(str(getattr(props, "uuid", ""))) if rank == 0 else None
    # untimed load so the clocks settle under load before the timed region
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
    h0 = time.perf_counter()
    ev0.record(stream)
    for i in range(args.steps):
        one(i)
    ev1.record(stream)
    if clk:
        clk.mark()  # the GPU is still running the steps just enqueued
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    dec.sync()  # raises on a recorded device-side timeout
    if world > 1:
        dist.barrier()
    ms_total = ev0.elapsed_time(ev1)
    clocks = clk.stop(h0, h1) if clk else None

    # per-step distribution: a second pass of K steps with an event after every step (an
    # event between two steps also ends the launch overlap between them, so these times
    # are those of steps run one after another without it)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        one(i)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    dec.sync()
    step_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]

    ms_total = max_over_ranks(ms_total, world, dev)
    ms_per_step = ms_total / args.steps
    value = job_steps_per_s(ms_per_step, world, args.tp)
    med, p10, p90 = step_percentiles(step_ms)

    # end to end through the host-buffer entry point: H2D x, step, D2H out, sync, every step,
    # on every rank; the slowest rank's wall time sets the job's rate
    e2e = None
    if TK == 1:
        xh = [torch.from_numpy(inp.x[t].view(np.int16)).view(torch.bfloat16).pin_memory() for t in range(T)]
        oh = torch.empty(B, shape.hidden, dtype=torch.float32).pin_memory()
        n_e2e = args.e2e_steps if args.e2e_steps > 0 else max(10, min(args.steps, 2000))
        ohs = [torch.empty(B, shape.hidden, dtype=torch.float32).pin_memory() for _ in range(2)]
        for i in range(3):
            dec.step_host(xh[i % T], ws[i % R], states[i % R], oh)
            dec.step_host_async(xh[i % T], ws[i % R], states[i % R], ohs[i % 2])
        dec.sync()
        if world > 1:
            dist.barrier()
        # pipelined: kda_decode_step_host_async every step (x in and out back on the handle's
        # copy stream, overlapping the neighbouring steps), one wait at the end
        t0 = time.perf_counter()
        for i in range(n_e2e):
            dec.step_host_async(xh[i % T], ws[i % R], states[i % R], ohs[i % 2])
        dec.sync()
        dt = max_over_ranks(time.perf_counter() - t0, world, dev)
        # blocking: kda_decode_step_host, which waits for its result every step
        t0 = time.perf_counter()
        for i in range(n_e2e):
            dec.step_host(xh[i % T], ws[i % R], states[i % R], oh)
        dtb = max_over_ranks(time.perf_counter() - t0, world, dev)
        e2e = {"value": job_steps_per_s(1000.0 * dt / n_e2e, world, args.tp), "unit": "steps/s",
               "h2d_bytes_per_step": int(xh[0].numel() * 2), "d2h_bytes_per_step": int(oh.numel() * 4),
               "steps": n_e2e, "call": "kda_decode_step_host_async every step, one kda_decode_sync at the end",
               "blocking": {"value": job_steps_per_s(1000.0 * dtb / n_e2e, world, args.tp), "unit": "steps/s",
                            "call": "kda_decode_step_host (waits for its result) every step"}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and TK == 1:
        rate, n, cores = oracle_rate(shape, inp, seqs=B, budget_s=args.cpu_seconds, max_steps=1000)
        rate1, n1, _ = oracle_rate(shape, inp, seqs=1, budget_s=min(5.0, args.cpu_seconds), max_steps=50, threads=1)
        cpu = {"value": rate, "unit": "steps/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
               "sample": f"{n} fp64 oracle decode steps of the same workload (batch {B}, rank-1 form, "
                         f"OpenMP on {cores} threads), about {args.cpu_seconds:.0f} s of CPU work",
               "single_thread": {"value": rate1, "unit": "steps/s",
                                 "sample": f"{n1} oracle steps of one sequence on 1 thread, scaled to "
                                           f"full-batch steps"}}

    dec.close()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = measured_peaks()
    hbm_peak = peaks.get("hbm_gbs")
    peak_src = "measured" if hbm_peak else "fallback"
    hbm_peak = float(hbm_peak or FALLBACK_HBM_GBS)
    ib = ideal_bytes(shape, B, tokens=TK)
    achieved = ib / (ms_per_step * 1e-3) / 1e9
    traffic = None
    tfile = os.path.join(ROOT, "profiles", f"traffic_{shape.name}.json")  # (a head shard has its own name)
    if os.path.exists(tfile):
        try:
            tj = json.load(open(tfile))
            if tj.get("engine") == engine and tj.get("kernel_rev") == kernel_rev():
                traffic = tj.get("dram_bytes_per_launch")
        except (OSError, ValueError):
            traffic = None
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "peak_source": f"{peak_src} copy bandwidth",
                "kernel": ("whole step (one persistent kernel)" if launches == 1 else
                           f"whole step ({launches} kernels)"),
                "algorithmic_bytes_per_launch": ib if launches == 1 else None,
                "algorithmic_bytes_per_step": ib}
    if prefill:
        # many rows per weight read: the projections are dense contractions on the tensor cores
        fl = prefill_flops(shape, B * TK)
        tpk = peaks.get("bf16_tflops")
        tsrc = "measured" if tpk else "fallback"
        tpk = float(tpk or FALLBACK_BF16_TFLOPS)
        ach = fl / (ms_per_step * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": ach, "peak": tpk, "unit": "TFLOP/s", "frac": ach / tpk,
                    "traffic": None, "peak_source": f"{tsrc} cuBLAS bf16 GEMM (burst)",
                    "kernel": f"whole step ({launches} own kernels + {lib_launches} cuBLASLt GEMMs)",
                    "algorithmic_flops_per_step": fl,
                    "note": "FLOPs of the projections (x W_q, W_k, W_v, W_b, W_a_down; W_a_up t; W_o o), each "
                            "counted once although it runs as hi + lo bf16 passes; the chunk recurrence's fp32 "
                            "work is not counted"}
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if args.tp else "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(full_shape, 1 if args.tp else world, R),
                       **({"tokens_per_step": TK} if TK > 1 else {}),
                       **({"parallelism": f"tp{world} (heads split over the ranks, {shape.num_heads} per rank; the out "
                                          f"all-reduce inside the fused kernel over peer memory)"}
                          if args.tp else {})),
        "tokens_per_s": value * B * TK,
        "step_us": {"median": med * 1e3, "p10": p10 * 1e3, "p90": p90 * 1e3,
                    "note": "second pass, an event after every step on the launching stream (rank 0); "
                            "the events also stop consecutive steps from overlapping"},
        "hbm_gbs": achieved, "hbm_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "engine": {1: "simple", 2: "fused"}.get(engine, str(engine)),
        **({"prefill": {"tokens": TK, "chunk": args.chunk or 32}} if prefill else {}),
        "roofline": roofline,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        **({"library_launches": lib_launches * args.steps} if lib_launches else {}),
        "cpu_baseline": cpu,
        "ideal_flops_per_step": ideal_flops(shape, B * TK),
    }
    print(json.dumps(line), flush=True)
    return 0


FUSED_SOURCES = ("common.cuh", "fused.cu", "fused.cuh", "schedule.cu", "sm100.cuh")


def kernel_rev() -> str:
    """Hash of the fused engine's sources: a stored ncu traffic figure is reported only for the
    kernel it measured."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_attention_layer_kda_b200", "csrc")
    for n in FUSED_SOURCES:
        for line in open(os.path.join(d, n)):
            code = line.split("//", 1)[0].strip()  # comments and layout do not change the kernel
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ launcher

def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(nproc: int, argv, port: int, limit_s: int):
    """torch.distributed.run command that starts `nproc` ranks of this script (one per GPU)."""
    return ["timeout", "-k", "60", str(limit_s), sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__)] + list(argv)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default="b8")
    ap.add_argument("--engine", type=int, default=0, help="0 auto, 1 simple, 2 fused")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-window", type=float, default=0.5,
                    help="seconds of untimed steps before the timed region, so clocks settle under load")
    ap.add_argument("--e2e-steps", type=int, default=0, help="steps of the host-buffer end-to-end loop")
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallel by heads over the N ranks (the out all-reduce inside the kernel); "
                         "default: data parallel over sequences")
    ap.add_argument("--tokens", type=int, default=1,
                    help="tokens per sequence in one step (multi-token verify through kda_decode_step_tokens)")
    ap.add_argument("--prefill", type=int, default=0, help="time kda_prefill of this many tokens per sequence")
    ap.add_argument("--chunk", type=int, default=0, help="prefill chunk (16, 32, 64; 0: the library default)")
    ap.add_argument("--launch-limit", type=int, default=900, help="seconds before a self-launched job is killed")
    ap.add_argument("--print-rank", action="store_true", help=argparse.SUPPRESS)  # launcher self-check
    return ap.parse_args(argv)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    args = parse_args(argv)
    args.warmup = max(3, args.warmup)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not under torchrun: start one rank per GPU and hand back their exit status
        return subprocess.call(launch_command(args.gpus, argv, free_port(), args.launch_limit))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: {world} ranks are running but --gpus is {args.gpus}; refusing to report", file=sys.stderr)
        return 2
    if args.print_rank:
        print(json.dumps({"rank": rank, "world_size": world, "local_rank": local_rank}), flush=True)
        return 0
    shape = I.CONFIGS[WORKLOADS[args.workload]]
    if args.impl == "reference":
        return run_reference(args, shape, rank, world)
    return run_ours(args, shape, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
