#!/usr/bin/env python
"""Benchmark of the ADMM-Q layer solve on B200.

Default workload: one Qwen3-8B-shaped decoder layer (its four solves: q/k/v
stacked 4096 -> 6144, o 4096 -> 4096, gate/up stacked 4096 -> 24576, down
12288 -> 4096; W3 g128 T = 100; 262144 calibration tokens each).  One step =
the hot path of those four solves on device-resident inputs, each:
  Gram X^T X (tcgen05, bf16 -> fp32)  ->  damping + diagonal scaling  ->
  C0' GEMM + RTN start  ->  T ADMM iterations (GEMM 1 + GEMM 2 with the fused
  projection / dual update, one launch)  ->  residuals + objective  ->  pack.
The one-time eigendecompositions (cuSOLVER, float64) are outside the step:
they run before the warm-up, are timed on their own and reported under
`eigh`.  Extra keys: the q_proj layer alone (`q_proj`) and its min/max grid
refresh (`by_grid`), the HBM-bound kernels (`stream_kernels`), the float64
oracle on a bounded sample (`cpu_baseline`).

Multi-GPU: layers are independent problems, so every rank solves its own
layer (seed = rank) with no collective in the data path ("scaling": "weak").

    python bench.py [--gpus N --steps K --warmup W --workload decoder|q_proj|... --grid minmax]
    python bench.py --impl reference   # the float64 CPU oracle on a bounded sample
    python bench.py --impl reference --workload q_proj --cpu-full [--cpu-threads 1]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from post_weight_quantization_10_b200 import dist as D  # noqa: E402
from post_weight_quantization_10_b200 import workloads  # noqa: E402

DTYPES = {"mixed": "f32 via tf32+bf16 split", "3xtf32": "f32 via 3xtf32",
          "f16": "f32 via fp16x3 split (power-of-two scaled)"}
METRIC = "ADMM-Q layer solve: iters/s, TFLOP/s vs tensor peak; Gram TFLOP/s; s/layer"
REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"],
                    bf16_sust=j.get("bf16_tflops_sustained", j["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# Source files each measured kernel is compiled and launched from (its
# launch geometry, e.g. the tile visiting order, is set in admmq.cu): its
# DRAM traffic figure (profiles/traffic.json) stands only while these are
# unchanged.
KERNEL_SOURCES = {
    "admm_loop": ["ptx.cuh", "gemm.cuh", "kernels.cuh", "admm_loop.cuh", "admmq.cu"],
    "project": ["ptx.cuh", "gemm.cuh", "kernels.cuh", "admmq.cu"],
    "pack": ["admmq.cu"],
}


def source_hash(kernel=None):
    """Short hash of the CUDA sources of `kernel` (all of them for None);
    matches the ncu captures in profiles/."""
    import hashlib
    csrc = os.path.join(ROOT, "post_weight_quantization_10_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or [f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))]
    per = [hashlib.sha1(open(os.path.join(csrc, f), "rb").read()).hexdigest() + "  " + f
           for f in sorted(names)]
    return hashlib.sha1(("\n".join(per) + "\n").encode()).hexdigest()[:12]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` (a preset name) from
    the committed ncu capture, or None when there is no capture of that pair
    or the kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)[f"{kernel}@{workload}"]
    except (OSError, KeyError, ValueError):
        return None
    return t["dram_bytes_per_launch"] if t["source_hash"] == source_hash(kernel) else None


def workload_desc(p, grid):
    return (f"{p.name}: d_in={p.d_in} d_out={p.d_out} n={p.n} W{p.bits} g{p.group} T={p.iters} "
            f"grid={grid} (Qwen3-8B-shaped synthetic layer, seed=rank)")


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """SM clock, power and throttle reasons from `nvidia-smi -lms 50`, started
    before the warm-up (its first sample takes a moment to arrive).  Only the
    samples whose timestamps fall inside the timed windows (host wall clock,
    begin() .. end(), taken after a device synchronize on both sides) are
    reported."""

    def __init__(self, gpu_index: int, interval_ms: int = 50):
        self.gpu = gpu_index
        self.interval = interval_ms
        self.proc = None
        self.path = None
        self.windows = []
        self._t0 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms",
                 str(self.interval), "-i", str(self.gpu)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def begin(self):
        self._t0 = time.time()

    def end(self):
        if self._t0 is not None:
            self.windows.append((self._t0, time.time()))
        self._t0 = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((t, float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if any(a <= r[0] <= b for a, b in self.windows)]
        if not inside:
            return None
        sm = [r[1] for r in inside]
        reasons = set()
        for r in inside:
            for name, val in zip(REASONS, r[3]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside),
                "window_s": round(sum(b - a for a, b in self.windows), 3)}


# ------------------------------------------------------------- our solver


class LayerRun:
    """Device-resident state of one layer solve through the C ABI binding."""

    def __init__(self, A, p, grid, seed, device, split="auto", scaling=True, schedule="fused",
                 rescale_dual=False, fit_on_w=False):
        self.A, self.p = A, p
        self.X, self.W = workloads.make_layer(p, seed=seed, device=device, w_dtype=torch.bfloat16)
        self.H = torch.empty((p.d_in, p.d_in), dtype=torch.float32, device=device)
        self.gram_ws = torch.empty(A.gram_workspace_bytes(p.n, p.d_in), dtype=torch.uint8,
                                   device=device)
        prm = A.Params(bits=p.bits, group=p.group, iters=p.iters, rho0=p.rho0, gamma=p.gamma,
                       lambda_rel=p.lambda_rel, grid=grid, split=split, scaling=scaling,
                       schedule=schedule, rescale_dual=rescale_dual, fit_on_w=fit_on_w)
        self.s = A.Solver(p.d_in, p.d_out, prm, device=device)
        self.packed = torch.empty((p.d_out, p.d_in * p.bits // 32), dtype=torch.int32,
                                  device=device)

    def setup_eigh(self):
        A = self.A
        A.build_hessian(self.X, self.H, workspace=self.gram_ws)
        self.s.prepare(self.H, self.W)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        self.s.eigh()
        torch.cuda.synchronize()
        return time.perf_counter() - t0

    def step(self, ev=None, X=None, W=None):
        """One layer solve; X / W default to the run's device-resident inputs.
        NVTX ranges name the phases (gram, scale_init, admm, finish_pack)
        inside a "solve" range, for profilers."""
        A, p = self.A, self.p
        X = self.X if X is None else X
        W = self.W if W is None else W
        nv = torch.cuda.nvtx
        phases = ["gram", "scale_init", "admm", "finish_pack"]

        def mark(k):
            if ev:
                ev[k].record()
            if k > 0:
                nv.range_pop()
            if k < 4:
                nv.range_push(phases[k])

        nv.range_push("solve")
        mark(0)
        A.build_hessian(X, self.H, workspace=self.gram_ws)
        mark(1)
        self.s.prepare(self.H, W)   # damping + scaling (eigenbasis from setup)
        self.s.init()
        mark(2)
        self.s.iterate(0, p.iters)
        mark(3)
        self.s.finish()
        A.pack(self.s.codes, p.bits, out=self.packed)
        mark(4)
        nv.range_pop()


def objective_report(A, run):
    """Objective of the solve just run next to its RTN start and GPTQ on the
    same layer (same H, same fixed min/max grid for RTN and GPTQ)."""
    p = run.p
    obj_admm = float(run.s.objective.cpu())
    run.s.init()
    run.s.finish(resid=False)
    obj_rtn = float(run.s.objective.cpu())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    g_codes, g_scale, g_zero = A.gptq(run.H, run.W, p.bits, p.group, p.lambda_rel)
    torch.cuda.synchronize()
    gptq_s = time.perf_counter() - t0
    obj_gptq = run.s.objective_of(g_codes, g_scale, g_zero)
    del g_codes, g_scale, g_zero
    return {"admm_q": obj_admm, "rtn": obj_rtn, "gptq": obj_gptq,
            "admm_over_rtn": obj_admm / obj_rtn, "admm_over_gptq": obj_admm / obj_gptq,
            "gptq_s": gptq_s}


class ShardRun(LayerRun):
    """One layer split over the ranks: this rank's block of calibration tokens
    and of output rows; H is the all-reduced sum of the ranks' partial Grams
    (the layer's one exchange step), every rank eigendecomposes it and solves
    its rows."""

    def __init__(self, A, p, grid, rank, world, device, split="auto", schedule="fused"):
        from post_weight_quantization_10_b200 import sharded
        X = workloads.make_activations(p, seed=0, device=device)
        W = workloads.make_weights(p, seed=0, device=device, dtype=torch.bfloat16)
        t0, t1 = sharded.block(p.n, world, rank)
        self.rows = sharded.block(p.d_out, world, rank)
        self.A, self.p, self.world = A, p, world
        self.X = X[t0:t1].contiguous()
        self.W = W[self.rows[0]:self.rows[1]].contiguous()
        del X, W
        torch.cuda.empty_cache()
        self.H = torch.empty((p.d_in, p.d_in), dtype=torch.float32, device=device)
        self.gram_ws = torch.empty(A.gram_workspace_bytes(self.X.shape[0], p.d_in),
                                   dtype=torch.uint8, device=device)
        prm = A.Params(bits=p.bits, group=p.group, iters=p.iters, rho0=p.rho0, gamma=p.gamma,
                       lambda_rel=p.lambda_rel, grid=grid, split=split, schedule=schedule)
        self.s = A.Solver(p.d_in, self.W.shape[0], prm, device=device)
        self.packed = torch.empty((self.W.shape[0], p.d_in * p.bits // 32), dtype=torch.int32,
                                  device=device)

    def _gram(self):
        self.A.build_hessian(self.X, self.H, workspace=self.gram_ws)
        if self.world > 1:
            torch.distributed.all_reduce(self.H, op=torch.distributed.ReduceOp.SUM)

    def setup_eigh(self):
        self._gram()
        self.s.prepare(self.H, self.W)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        self.s.eigh()
        torch.cuda.synchronize()
        return time.perf_counter() - t0

    def step(self, ev=None):
        mark = (lambda k: ev[k].record()) if ev else (lambda k: None)
        mark(0)
        self._gram()
        mark(1)
        self.s.prepare(self.H, self.W)
        self.s.init()
        mark(2)
        self.s.iterate(0, self.p.iters)
        mark(3)
        self.s.finish()
        self.A.pack(self.s.codes, self.p.bits, out=self.packed)
        mark(4)


def run_sharded(args, rank, world, device):
    """One layer over all ranks (strong scaling): value = ADMM iterations of
    the whole layer per second, from the slowest rank's step time."""
    from post_weight_quantization_10_b200 import admmq as A
    A.lib()
    p = workloads.PRESETS[args.workload]
    if args.tokens:
        p = workloads.scaled(p, args.tokens, p.d_in, p.d_out)
    run = ShardRun(A, p, args.grid, rank, world, device, split=args.split, schedule=args.schedule)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    eigh_s = run.setup_eigh()
    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()
    dist_barrier(world)
    torch.cuda.synchronize()
    n0 = A.launch_count()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    clocks.begin()
    a.record()
    for k in range(args.steps):
        run.step(evs[k])
    b.record()
    torch.cuda.synchronize()
    clocks.end()
    dist_barrier(world)
    clk = clocks.stop()
    ms = dist_max(a.elapsed_time(b), world, device)
    phase = np.zeros(4)
    for e in evs:
        phase += [e[i].elapsed_time(e[i + 1]) for i in range(4)]
    phase /= args.steps
    obj = D.sum_over_ranks(float(run.s.objective.cpu()), world, device)
    if rank != 0:
        return None
    return {
        "metric": METRIC, "value": p.iters * args.steps / (ms / 1e3), "unit": "iters/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None,
        "dtype": DTYPES[run.s.split],
        "data": "synthetic (seeded Qwen3-8B-shaped activations and weights; no dataset)",
        "config": {"workload": workload_desc(p, args.grid) + " (one layer split over the ranks)",
                   "parallelism": f"tokens and output rows split over {world} ranks, "
                                  "H all-reduced", "split": run.s.split,
                   "l2": "inputs larger than L2"},
        "s_per_layer": ms / 1e3 / args.steps, "eigh_s": eigh_s,
        "phase_ms_rank0": {"gram_allreduce": phase[0], "scale_init": phase[1], "admm": phase[2],
                           "finish_pack": phase[3]},
        "objective": obj, "gpu_launches": A.launch_count() - n0, "clocks": clk,
    }


# Tensor work per fp32-accurate product, in bf16-MMA units (dense tf32 runs
# at half the bf16 rate, nominal 1.1 vs 2.25 PFLOP/s): 3xTF32 = three tf32
# MMAs = 6; fp16 x3 = three full-rate fp16 MMAs = 3; mixed split = one tf32
# MMA (2) + one bf16 MMA over the doubled K of the correction rows (2) = 4.
# Peak of a split = bf16 peak / that.
PER_PRODUCT = {"mixed": 4.0, "3xtf32": 6.0, "f16": 3.0}


def split_peak(split, pk):
    return pk["bf16_sust"] / PER_PRODUCT[split]


def fused_stats(run):
    """(ms per fused launch, algorithmic flops per launch, launches) of the
    timed launches of `run` (the fused schedule: one launch runs GEMM 1 and
    GEMM 2 of all iterations of the solve, 4 d^2 m flops per iteration)."""
    gemm_ms, gemm_n, gemm_iters = run.s.get_timing()
    p = run.p
    n = max(gemm_n[0], 1)
    return gemm_ms[0] / n, 4.0 * p.d_in * p.d_in * p.d_out * gemm_iters / n, gemm_n[0]


def measure_layer(A, p, grid, seed, device, steps, warmup, split="auto", schedule="fused",
                  objective=True, clocks=None):
    """One layer preset timed like the main line (device-resident inputs,
    CUDA events), for the extra keys: iterations/s, fused-launch time and its
    roofline, Gram rate, objective next to RTN and GPTQ."""
    pk = peaks()
    run = LayerRun(A, p, grid, seed=seed, device=device, split=split, schedule=schedule)
    eigh_s = run.setup_eigh()
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize()
    run.s.set_timing(True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.begin()
    a.record()
    for k in range(steps):
        run.step(evs[k])
    b.record()
    torch.cuda.synchronize()
    if clocks:
        clocks.end()
    run.s.check()
    ms = a.elapsed_time(b) / steps
    ph = np.mean([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in evs], axis=0)
    launch_ms, flops, _ = fused_stats(run)
    run.s.set_timing(False)
    ach = flops / (launch_ms / 1e3) / 1e12
    peak = split_peak(run.s.split, pk)
    out = {"workload": workload_desc(p, grid), "split": run.s.split,
           "iters_per_s": p.iters / (ms / 1e3), "ms_per_step": ms,
           "fused_launch_ms": launch_ms,
           "admm_tflops_fp32_accurate": ach, "frac_of_split_peak": ach / peak,
           "gram_tflops": float(p.n) * p.d_in * (p.d_in + 1) / (ph[0] / 1e3) / 1e12,
           "phase_ms": {"gram": ph[0], "scale_init": ph[1], "admm": ph[2], "finish_pack": ph[3]},
           "eigh_s": eigh_s}
    if objective:
        out["objective"] = objective_report(A, run)
    del run
    torch.cuda.empty_cache()
    return out


def eigh_overlap(runs):
    """The layer's setup and solves, timed three ways (host timers around
    device-synchronised work): one after the other (each solve's prepare +
    eigh, then its solve); with every eigendecomposition on a second stream
    from a host thread, each solve waiting only for its own; and with only
    the largest one on the side stream while the others run in order
    (pipeline.solve_overlapped, whose schedule the critical path favours)."""
    import threading
    from post_weight_quantization_10_b200.pipeline import solve_overlapped
    dev = runs[0].X.device

    def eig(r, stream=None):
        r.s.prepare(r.H, r.W, stream)
        r.s.eigh(stream)

    def solve(r, stream=None):
        r.s.solve(stream)

    for r in runs:
        r.s.set_timing(False)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for r in runs:
        eig(r)
        solve(r)
    torch.cuda.synchronize()
    serial = time.perf_counter() - t0
    sA = torch.cuda.Stream(device=dev)
    sB = torch.cuda.Stream(device=dev)
    ready = [threading.Event() for _ in runs]
    errors = []

    def worker():
        try:
            torch.cuda.set_device(dev)
            for i, r in enumerate(runs):
                eig(r, sA)
                ready[i].set()
        except Exception as e:  # reported after the join
            errors.append(e)
            for ev in ready:
                ev.set()

    torch.cuda.synchronize()
    t0 = time.perf_counter()
    th = threading.Thread(target=worker)
    th.start()
    for i, r in enumerate(runs):
        ready[i].wait()
        ev = torch.cuda.Event()
        ev.record(sA)
        sB.wait_event(ev)
        solve(r, sB)
    th.join()
    torch.cuda.synchronize()
    if errors:
        raise errors[0]
    all_side = time.perf_counter() - t0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    solve_overlapped([(r.s, r.H, r.W) for r in runs])
    torch.cuda.synchronize()
    largest_side = time.perf_counter() - t0
    for r in runs:
        r.s.check()
    return {"serial_s": serial, "overlapped_s": largest_side, "all_eigh_on_side_stream_s": all_side,
            "note": "one decoder layer's four (prepare + eigh, solve): in order; with the largest "
                    "eigendecomposition on a second stream while the other three solves run "
                    "(overlapped_s, pipeline.solve_overlapped); and with every "
                    "eigendecomposition on the second stream"}


def run_decoder(args, rank, world, device):
    """One Qwen3-8B-shaped decoder layer per rank: its four solves (q/k/v and
    gate/up stacked on their shared inputs) are one step.  The value is the
    seconds per decoder layer of the whole job (slowest rank's time over the
    layers all ranks solved)."""
    from post_weight_quantization_10_b200 import admmq as A
    A.lib()
    pk = peaks()
    bits = args.bits or 3
    specs = []
    for label, p, seed in workloads.decoder_layer(bits):
        if args.solve and label != args.solve:
            continue
        if args.tokens:
            p = workloads.scaled(p, args.tokens, p.d_in, p.d_out)
        specs.append((label, p, seed))
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    runs = [LayerRun(A, p, args.grid, seed=seed + 1000 * rank, device=device, split=args.split,
                     schedule=args.schedule) for _, p, seed in specs]
    eigh_s = [r.setup_eigh() for r in runs]
    for _ in range(args.warmup):
        for r in runs:
            r.step()
    torch.cuda.synchronize()

    # ---- device-resident timed region
    dist_barrier(world)
    torch.cuda.synchronize()
    for r in runs:
        r.s.set_timing(True)
    n0 = A.launch_count()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in runs]
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.begin()
    torch.cuda.nvtx.range_push("timed")
    t_start.record()
    for k in range(args.steps):
        for i, r in enumerate(runs):
            r.step(evs[k][i])
    t_end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clocks.end()
    dist_barrier(world)
    launches = A.launch_count() - n0
    for r in runs:
        r.s.check()   # a timed-out wait or an fp16 range overflow invalidates the run
    ms = t_start.elapsed_time(t_end)
    ms_max = dist_max(ms, world, device)
    phases = np.zeros((len(runs), 4))
    for k in range(args.steps):
        for i in range(len(runs)):
            e = evs[k][i]
            phases[i] += [e[j].elapsed_time(e[j + 1]) for j in range(4)]
    phases /= args.steps
    fused = [fused_stats(r) for r in runs]
    for r in runs:
        r.s.set_timing(False)

    e2e = None if args.no_e2e else run_e2e(A, runs, args, world, device)
    objectives = [objective_report(A, r) for r in runs]
    overlap = None if args.no_eigh_overlap else eigh_overlap(runs)

    solves = []
    for (label, p, _), r, ph, (lms, lfl, _), ob, es in zip(specs, runs, phases, fused,
                                                           objectives, eigh_s):
        ach = lfl / (lms / 1e3) / 1e12
        solves.append({
            "solve": label, "d_in": p.d_in, "d_out": p.d_out, "bits": p.bits, "iters": p.iters,
            "split": r.s.split, "s": float(ph.sum()) / 1e3,
            "iters_per_s": p.iters / (ph[2] / 1e3),
            "fused_launch_ms": lms, "admm_tflops_fp32_accurate": ach,
            "frac_of_split_peak": ach / split_peak(r.s.split, pk),
            "gram_tflops": float(p.n) * p.d_in * (p.d_in + 1) / (ph[0] / 1e3) / 1e12,
            "phase_ms": {"gram": ph[0], "scale_init": ph[1], "admm": ph[2], "finish_pack": ph[3]},
            "eigh_s": es, "objective": ob})
    splits = sorted({r.s.split for r in runs})
    launch_ms = sum(f[0] for f in fused)
    launch_flops = sum(f[1] for f in fused)
    achieved = launch_flops / (launch_ms / 1e3) / 1e12   # flops-weighted over the 4 launches
    peak = split_peak(splits[0], pk)
    gram_flops = sum(float(p.n) * p.d_in * (p.d_in + 1) for _, p, _ in specs)
    layers = args.steps * world
    s_layer = ms_max / 1e3 / layers
    tot = {k: sum(o[k] for o in objectives) for k in ("admm_q", "rtn", "gptq")}
    line = {
        "metric": METRIC,
        "value": s_layer, "unit": "s/layer",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None,
        "dtype": " / ".join(DTYPES[x] for x in splits),
        "data": "synthetic (seeded Qwen3-8B-shaped activations and weights; no dataset)",
        "config": {"workload": ("Qwen3-8B-shaped decoder layer (four solves): qkv 4096->6144, "
                                "o 4096->4096, gate_up 4096->24576, down 12288->4096; "
                                "n=%d tokens each; W%d g128 T=%d grid=%s" % (
                                    specs[0][1].n, bits, specs[0][1].iters, args.grid))
                               + (" [only the %s solve]" % args.solve if args.solve else ""),
                   "parallelism": f"independent decoder layers x{world}",
                   "l2": "inputs larger than L2 (X is %.1f GiB per step)" % (
                       sum(p.n * p.d_in * 2 for _, p, _ in specs) / 2**30),
                   "eigh": "one-time setup outside the step (eigh)",
                   "split": "/".join(splits), "schedule": args.schedule},
        "iters_per_s_layer": specs[0][1].iters * layers / (ms_max / 1e3),
        "gram_tflops": gram_flops / (phases[:, 0].sum() / 1e3) / 1e12,
        "phase_ms": {"gram": phases[:, 0].sum(), "scale_init": phases[:, 1].sum(),
                     "admm": phases[:, 2].sum(), "finish_pack": phases[:, 3].sum()},
        "roofline": {"kernel": "admm_loop", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": measured_traffic("admm_loop", f"decoder_w{bits}"),
                     "launches_per_step": len(runs),
                     "peak_note": "bf16 dense %s sustained %.1f TF/s / %d (bf16-MMA units of "
                                  "tensor work per fp32-accurate product, %s split); achieved = "
                                  "the four solves' algorithmic flops / their fused-launch time" % (
                                      pk["src"], pk["bf16_sust"], PER_PRODUCT[splits[0]],
                                      splits[0])},
        "solves": solves,
        "eigh": {"per_solve_s": {x["solve"]: x["eigh_s"] for x in solves},
                 "total_s": sum(eigh_s), "overlap": overlap},
        "s_per_layer_with_eigh": s_layer + sum(eigh_s),
        "qwen3_8b_36_layers_h": (s_layer + sum(eigh_s)) * 36 / 3600,
        "objective": dict(tot, admm_over_rtn=tot["admm_q"] / tot["rtn"],
                          admm_over_gptq=tot["admm_q"] / tot["gptq"],
                          note="sums over the four solves of 1/2 Tr((D - W_hat)^T H (D - W_hat)), "
                               "H = X^T X + lambda I; RTN and GPTQ on the min/max grid of W_hat, "
                               "ADMM-Q with its refreshed grid; per solve under solves"),
        "gpu_launches": launches,
        "e2e": e2e,
    }
    del runs
    torch.cuda.empty_cache()
    if not args.no_extra:
        qp = workloads.PRESETS["q_proj"]
        if args.tokens:
            qp = workloads.scaled(qp, args.tokens, qp.d_in, qp.d_out)
        ksteps = max(2, min(args.steps, 5))
        line["q_proj"] = measure_layer(A, qp, args.grid, rank, device, ksteps, 2, args.split,
                                       args.schedule)
        other = "minmax" if args.grid != "minmax" else "lsq"
        line["by_grid"] = {
            args.grid: {k: line["q_proj"][k] for k in ("iters_per_s", "fused_launch_ms",
                                                       "frac_of_split_peak", "objective")},
            other: measure_layer(A, qp, other, rank, device, ksteps, 2, args.split,
                                 args.schedule)}
    line["clocks"] = clocks.stop()
    if not args.no_stream_kernels:
        line["stream_kernels"] = stream_kernels(A, args.grid, device)
    if rank != 0:
        return None
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline([p for _, p, _ in specs], args.grid, "s/layer")
    return line


def run_ours(args, rank, world, device):
    from post_weight_quantization_10_b200 import admmq as A
    A.lib()
    p = workloads.PRESETS[args.workload]
    if args.tokens:
        p = workloads.scaled(p, args.tokens, p.d_in, p.d_out)
    run = LayerRun(A, p, args.grid, seed=rank, device=device, split=args.split,
                   scaling=not args.no_scaling, schedule=args.schedule,
                   rescale_dual=args.rescale_dual, fit_on_w=args.fit_on_w)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    eigh_s = run.setup_eigh()
    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()

    # ---- device-resident timed region
    dist_barrier(world)
    torch.cuda.synchronize()
    run.s.set_timing(True)
    n0 = A.launch_count()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.begin()
    torch.cuda.nvtx.range_push("timed")
    t_start.record()
    for k in range(args.steps):
        run.step(evs[k])
    t_end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clocks.end()
    dist_barrier(world)
    launches = A.launch_count() - n0
    clk = clocks.stop()
    run.s.check()   # a timed-out wait or an fp16 range overflow invalidates the run
    ms = t_start.elapsed_time(t_end)
    gemm_ms, gemm_n, gemm_iters = run.s.get_timing()
    run.s.set_timing(False)
    phase = np.zeros(4)
    for e in evs:
        phase += [e[i].elapsed_time(e[i + 1]) for i in range(4)]
    phase /= args.steps
    ms_max = dist_max(ms, world, device)

    # ---- end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(A, [run], args, world, device)

    # objective 1/2 Tr((D - W_hat)^T H (D - W_hat)) of the solve just timed,
    # next to its RTN start and GPTQ on the same layer
    obj = objective_report(A, run)

    if rank != 0:
        return None
    pk = peaks()
    d, m, n, T = p.d_in, p.d_out, p.n, p.iters
    layers = args.steps * world
    iters_per_s = T * layers / (ms_max / 1e3)
    flops_iter = 4.0 * d * d * m
    admm_ms = phase[2]
    gram_flops = float(n) * d * (d + 1)
    if gemm_n[1] == 0:
        # fused schedule: one launch runs GEMM 1 and GEMM 2 of every iteration
        # of the solve (4 d^2 m flops per iteration)
        kname = "admm_loop"
        avg_ms = gemm_ms[0] / max(gemm_n[0], 1)
        flops_launch = flops_iter * gemm_iters / max(gemm_n[0], 1)
        per_launch = {"admm_loop": avg_ms, "iters_per_launch": gemm_iters / max(gemm_n[0], 1)}
    else:
        # dominant kernel: GEMM 1 or GEMM 2 (same algorithmic flops, 2 d^2 m each)
        k = 0 if gemm_ms[0] >= gemm_ms[1] else 1
        kname = ["gemm1_eigscale", "gemm2_project"][k]
        avg_ms = gemm_ms[k] / max(gemm_n[k], 1)
        flops_launch = 2.0 * d * d * m
        per_launch = {"gemm1_eigscale": gemm_ms[0] / max(gemm_n[0], 1),
                      "gemm2_project": gemm_ms[1] / max(gemm_n[1], 1)}
    achieved = flops_launch / (avg_ms / 1e3) / 1e12
    split = run.s.split
    per_product = PER_PRODUCT[split]
    peak_split = split_peak(split, pk)
    line = {
        "metric": METRIC,
        "value": iters_per_s,
        "unit": "iters/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPES[split],
        "data": "synthetic (seeded Qwen3-8B-shaped activations and weights; no dataset)",
        "config": {"workload": workload_desc(p, args.grid)
                   + (" Sigma=I (unscaled ablation)" if args.no_scaling else "")
                   + (" dual rescaled by rho_t/rho_t+1" if args.rescale_dual else "")
                   + (" grid fitted on W~" if args.fit_on_w else ""),
                   "parallelism": f"independent layers x{world}",
                   "l2": "inputs larger than L2 (X is %.1f GiB)" % (n * d * 2 / 2**30),
                   "eigh": "one-time setup outside the step (eigh_s)",
                   "split": split, "schedule": args.schedule},
        "s_per_layer": ms_max / 1e3 / args.steps,
        "s_per_layer_with_eigh": ms_max / 1e3 / args.steps + eigh_s,
        "eigh_s": eigh_s,
        "phase_ms": {"gram": phase[0], "scale_init": phase[1], "admm": phase[2],
                     "finish_pack": phase[3]},
        "admm_iters_per_s": T / (admm_ms / 1e3),
        "admm_tflops_fp32_accurate": flops_iter * T / (admm_ms / 1e3) / 1e12,
        "gram_tflops": gram_flops / (phase[0] / 1e3) / 1e12,
        "ms_per_launch": per_launch,
        "roofline": {"kernel": kname, "bound": "tensor",
                     "achieved": achieved, "peak": peak_split, "unit": "TFLOP/s",
                     "frac": achieved / peak_split,
                     "traffic": measured_traffic(kname, args.workload),
                     "peak_note": "bf16 dense %s sustained %.1f TF/s / %d (bf16-MMA units of tensor "
                                  "work per fp32-accurate product, %s split)" % (
                                      pk["src"], pk["bf16_sust"], per_product, split)},
        "objective": dict(obj, note="1/2 Tr((D - W_hat)^T H (D - W_hat)), H = X^T X + lambda I; "
                                    "RTN and GPTQ on the min/max grid of W_hat, ADMM-Q with its "
                                    "refreshed grid"),
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
    }
    if not args.no_stream_kernels:
        line["stream_kernels"] = stream_kernels(A, args.grid, device)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline([p], args.grid, "iters/s")
    return line


def stream_kernels(A, grid, device, reps=10):
    """HBM-bound kernels timed on their own, on buffers larger than L2: the
    standalone projection (the fused epilogue's float32 arithmetic reading W~
    from memory) and the b-bit pack.  The projection writes P in the fp16
    split, the encoding the solve uses at this shape (d_in >= 2048); its
    algorithmic bytes per element: W~ 4, V 4 + 4, codes 1 + 1, P planes 2 + 2
    (18).  `project_by_grid` times every grid refresh in that encoding, and
    the least-squares one also in the mixed encoding (P planes 4 + 4, 22
    bytes).  The pack: codes 1 + b/8 bytes per element."""
    pk = peaks()
    m, d, g, bits = 25600, 5120, 128, 3          # the up_proj 32B layer shape
    gen = torch.Generator(device=device).manual_seed(7)
    wt = torch.randn((m, d), generator=gen, device=device) * 0.02
    V = torch.randn((m, d), generator=gen, device=device) * 0.002
    sig = torch.rand(d, generator=gen, device=device) + 0.5
    rsig = 1.0 / sig
    hd = rsig * rsig
    L = (1 << bits) - 1
    codes = torch.randint(0, L + 1, (m, d), generator=gen, device=device, dtype=torch.uint8)
    scale = torch.full((m, d // g), 0.01, device=device)
    zero = torch.full((m, d // g), 3.0, device=device)
    # row scales of the fp16 split: 2^e with |row| 2^e in [2^9, 2^10)
    rows = torch.linalg.vector_norm(wt, dim=1)
    row_scale = torch.exp2(torch.ceil(9.0 - torch.log2(rows)))
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    phi = torch.empty((m, d), device=device)     # mixed: fp32 plane, bf16 correction rows
    plo = torch.empty((m, 2 * d), dtype=torch.int16, device=device)
    f16_hi = torch.empty((m, d), dtype=torch.int16, device=device)
    f16_lo = torch.empty((m, d), dtype=torch.int16, device=device)
    resid = torch.zeros(2, dtype=torch.float64, device=device)
    big = torch.randint(0, L + 1, (4 * m, d), generator=gen, device=device, dtype=torch.uint8)
    packed = torch.empty((4 * m, d * bits // 32), dtype=torch.int32, device=device)

    def proj(gr, split):
        if split == "f16":
            return lambda: A.project(wt, V, sig, rsig, hd, bits, g, gr, codes, scale, zero,
                                     f16_hi, f16_lo, resid=resid, split="f16",
                                     row_scale=row_scale, range_flag=flag)
        return lambda: A.project(wt, V, sig, rsig, hd, bits, g, gr, codes, scale, zero,
                                 phi, plo, resid=resid, split="mixed")

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def entry(ms, nbytes, shape, traffic):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"shape": shape, "bits": bits, "alg_bytes": nbytes, "ms": ms, "gbs": gbs,
                "frac_hbm": gbs / pk["hbm"], "traffic": traffic}

    out = {}
    out["project"] = entry(timed(proj(grid, "f16")), 18.0 * m * d, [m, d],
                           measured_traffic("project", "stream") if grid == "lsq" else None)
    out["project"].update(grid=grid, split="f16")
    by = {}
    for gr, split, nb in (("lsq", "f16", 18.0), ("minmax", "f16", 18.0), ("frozen", "f16", 18.0),
                          ("mse", "f16", 18.0), ("lsq", "mixed", 22.0)):
        e = entry(timed(proj(gr, split)), nb * m * d, [m, d], None)
        by[f"{gr}/{split}"] = {k: e[k] for k in ("ms", "gbs", "frac_hbm", "alg_bytes")}
    out["project_by_grid"] = by
    out["pack"] = entry(timed(lambda: A.pack(big, bits, out=packed)), (1 + bits / 8) * 4 * m * d,
                        [4 * m, d], measured_traffic("pack", "stream"))
    if int(flag.item()) != 0:
        raise RuntimeError("stream projection: fp16 range flag set")
    del wt, V, codes, phi, plo, f16_hi, f16_lo, big, packed
    torch.cuda.empty_cache()
    return out


def run_e2e(A, runs, args, world, device):
    """The step through the public API from pinned host buffers: every step
    copies each solve's X and W_hat to the device and reads its codes, packed
    words, grid and objective back.  Each solve's inputs are copied on a
    second stream while the solve before it runs (pipeline.InputPipeline,
    one device slot per solve); the first copy of the run is not
    overlapped."""
    from post_weight_quantization_10_b200.pipeline import InputPipeline
    copy_stream = torch.cuda.Stream(device=device)
    hosts, outs, pipes = [], [], []
    h2d = d2h = 0
    for run in runs:
        Xh = torch.empty(run.X.shape, dtype=run.X.dtype, pin_memory=True)
        Xh.copy_(run.X)
        Wh = torch.empty(run.W.shape, dtype=run.W.dtype, pin_memory=True)
        Wh.copy_(run.W)
        o = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
             for t in (run.s.codes, run.packed, run.s.scale, run.s.zero, run.s.objective)]
        hosts.append([Xh, Wh])
        outs.append(o)
        h2d += sum(t.numel() * t.element_size() for t in (Xh, Wh))
        d2h += sum(t.numel() * t.element_size() for t in o)
        pipes.append(InputPipeline([Xh, Wh], device, slots=1 if len(runs) > 1 else 2,
                                   copy_stream=copy_stream))
    nr = len(runs)

    def steps(k):
        slot = pipes[0].prefetch(hosts[0])
        for j in range(k * nr):
            i = j % nr
            run = runs[i]
            X, W = pipes[i].acquire(slot)
            nxt = pipes[(i + 1) % nr].prefetch(hosts[(i + 1) % nr]) if j + 1 < k * nr else None
            run.step(X=X, W=W)
            pipes[i].release(slot)
            for dst, src in zip(outs[i], (run.s.codes, run.packed, run.s.scale, run.s.zero,
                                          run.s.objective)):
                dst.copy_(src, non_blocking=True)
            slot = nxt

    steps(1)
    torch.cuda.synchronize()
    dist_barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    steps(args.steps)
    b.record()
    torch.cuda.synchronize()
    dist_barrier(world)
    for run in runs:
        run.s.check()
    ms = dist_max(a.elapsed_time(b), world, device)
    del pipes
    torch.cuda.empty_cache()
    layers = args.steps * world
    if nr == 1:
        value, unit = runs[0].p.iters * layers / (ms / 1e3), "iters/s"
    else:
        value, unit = ms / 1e3 / layers, "s/layer"
    return {"value": value, "unit": unit,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "s_per_layer": ms / 1e3 / args.steps,
            "overlap": "each solve's inputs are copied on a second stream during the solve "
                       "before it (the first copy is not overlapped)"}


# --------------------------------------------------- CPU oracle (baseline)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 0) for i in info), default=None)
    except Exception:
        return None


CPU_TOKENS, CPU_ROWS = 2048, 512


def sample_desc(p, tokens=CPU_TOKENS, rows=CPU_ROWS):
    return (f"Gram of {min(tokens, p.n)} of {p.n} tokens + 1 of {p.iters} ADMM iterations on "
            f"{min(rows, p.d_out)} of {p.d_out} output rows at d_in={p.d_in}, extrapolated "
            f"linearly in n and d_out (eigh excluded, as on the GPU)")


def cpu_sample(p, grid, seed=0, tokens=CPU_TOKENS, rows=CPU_ROWS):
    """Time the float64 oracle on a bounded sample of one solve: the Gram of
    `tokens` calibration tokens and one ADMM iteration (W-update, projection,
    dual update) on `rows` output rows at the full d_in; extrapolate linearly
    to the step (n tokens, d_out rows, T iterations: the Gram is linear in n,
    an iteration linear in d_out)."""
    from oracle import admmq_oracle as O
    rng = np.random.default_rng(seed)
    d, m = p.d_in, p.d_out
    ns, ms = min(tokens, p.n), min(rows, m)
    Xs = rng.standard_normal((ns, d)).astype(np.float32)
    t0 = time.perf_counter()
    O.gram(Xs)
    t_gram = (time.perf_counter() - t0) * (p.n / ns)
    Q = rng.standard_normal((d, d)) / np.sqrt(d)
    lam = np.abs(rng.standard_normal(d)) + 0.1
    B = rng.standard_normal((d, ms)) * 0.02
    Dt = rng.standard_normal((d, ms)) * 0.02
    Vt = rng.standard_normal((d, ms)) * 0.002
    sigma = np.abs(rng.standard_normal(d)) * 0.01 + 0.01
    hdiag = (1.0 / sigma ** 2).astype(np.float32)
    s_prev = np.full((d // p.group, ms), 0.01, np.float32)
    z_prev = np.full((d // p.group, ms), 3.0, np.float32)
    t0 = time.perf_counter()
    Wt = O.w_update(Q, lam, B, 0.1, Dt, Vt)
    Y = sigma[:, None] * (Wt + Vt)
    _, _, _, D = O.project(Y, p.bits, p.group, grid, hdiag, s_prev, z_prev)
    Vt = Vt + Wt - D / sigma[:, None]
    t_iter = (time.perf_counter() - t0) * (m / ms)
    step_s = t_gram + p.iters * t_iter
    return dict(t_gram=t_gram, t_iter=t_iter, step_s=step_s, iters_per_s=p.iters / step_s,
                sample=sample_desc(p, tokens, rows))


def _cpu_threads(n):
    """Limit the BLAS pools to n threads (0: leave them); returns the limiter."""
    if not n:
        return None
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=n)


def _cores():
    return {"blas_threads": _blas_threads(), "host_cpus": os.cpu_count()}


def cpu_baseline(presets, grid, unit, reps=4):
    """The oracle as it stands on a bounded sample of the step's solves
    (cpu_sample each, summed over the solves), `reps` times; seconds per step
    or iterations per second."""
    vals = [sum(cpu_sample(p, grid, seed=r)["step_s"] for p in presets) for r in range(reps)]
    step_s = float(np.median(vals))
    c = _cores()
    value = step_s if unit == "s/layer" else presets[0].iters / step_s
    return {"value": value, "unit": unit, "cores": c["blas_threads"] or c["host_cpus"],
            "host_cpus": c["host_cpus"], "kind": "oracle",
            "sample": "per solve: " + sample_desc(presets[0]).replace(
                f"d_in={presets[0].d_in}", "full d_in") + (
                "; summed over the %d solves, median of %d" % (len(presets), reps)),
            "s_per_layer": step_s}


def cpu_full(p, grid, seed=0):
    """The oracle's whole solve of one layer preset, no extrapolation: Gram
    over all n tokens (8192-token chunks), damping and scaling, eigh, T
    iterations, objective; wall-clock seconds of each phase."""
    from oracle import admmq_oracle as O
    rng = np.random.default_rng(seed)
    d, m = p.d_in, p.d_out
    t0 = time.perf_counter()
    G = np.zeros((d, d))
    for r0 in range(0, p.n, 8192):
        Xc = rng.standard_normal((min(8192, p.n - r0), d)).astype(np.float32)
        G += O.gram(Xc)
    t_gram = time.perf_counter() - t0
    H, _ = O.damping(G, p.lambda_rel)
    W = rng.standard_normal((d, m)) * p.w_std
    t0 = time.perf_counter()
    eig = np.linalg.eigh(O.diagonal_scaling(H)[1])
    t_eigh = time.perf_counter() - t0
    t0 = time.perf_counter()
    res = O.admm_q(H, W, p.bits, p.group, p.iters, rho0=p.rho0, gamma=p.gamma, grid=grid, eig=eig)
    t_iters = time.perf_counter() - t0
    return {"gram_s": t_gram, "eigh_s": t_eigh, "iters_s": t_iters,
            "step_s": t_gram + t_iters, "iters_per_s": p.iters / t_iters,
            "objective": res["objective"]}


def run_reference_decoder(args, world):
    """The oracle on the decoder-layer workload: the bounded sample of each of
    the four solves, summed (seconds per decoder layer)."""
    bits = args.bits or 3
    presets = [p for _, p, _ in workloads.decoder_layer(bits)]
    for _ in range(args.warmup):
        cpu_sample(presets[0], args.grid)
    vals = [sum(cpu_sample(p, args.grid, seed=k)["step_s"] for p in presets)
            for k in range(args.steps)]
    value = float(np.mean(vals))
    c = _cores()
    sample = "per solve: " + sample_desc(presets[0]).replace(
        f"d_in={presets[0].d_in}", "full d_in") + "; summed over the four solves"
    return {"impl": "reference", "metric": METRIC,
            "value": value, "unit": "s/layer", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": value * 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "Qwen3-8B-shaped decoder layer (four solves): qkv 4096->6144, "
                                   "o 4096->4096, gate_up 4096->24576, down 12288->4096; "
                                   "n=262144 tokens each; W%d g128 T=%d grid=%s" % (
                                       bits, presets[0].iters, args.grid)},
            "cpu_baseline": {"value": value, "unit": "s/layer",
                             "cores": c["blas_threads"] or c["host_cpus"],
                             "host_cpus": c["host_cpus"], "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "s/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    lim = _cpu_threads(args.cpu_threads)
    try:
        if args.workload == "decoder":
            return run_reference_decoder(args, world)
        p = workloads.PRESETS[args.workload]
        c = _cores()
        if args.cpu_full:
            r = cpu_full(p, args.grid)
            return {"impl": "reference", "metric": METRIC, "value": r["iters_per_s"],
                    "unit": "iters/s", "n_gpus": world, "steps": 1, "warmup": 0,
                    "ms_per_step": r["step_s"] * 1e3, "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "config": {"workload": workload_desc(p, args.grid)},
                    "cpu_full": r, "cores": c["blas_threads"] or c["host_cpus"],
                    "host_cpus": c["host_cpus"],
                    "sample": "the whole solve, no extrapolation (eigh timed apart)"}
        for _ in range(args.warmup):
            cpu_sample(p, args.grid)
        vals = [cpu_sample(p, args.grid, seed=k) for k in range(args.steps)]
        step_s = float(np.mean([v["step_s"] for v in vals]))
        value = p.iters / step_s
        return {"impl": "reference", "metric": METRIC, "value": value, "unit": "iters/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload_desc(p, args.grid)},
                "cpu_baseline": {"value": value, "unit": "iters/s",
                                 "cores": c["blas_threads"] or c["host_cpus"],
                                 "host_cpus": c["host_cpus"], "kind": "oracle",
                                 "sample": vals[0]["sample"]},
                "e2e": {"value": value, "unit": "iters/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    finally:
        if lim is not None:
            lim.restore_original_limits()


# ------------------------------------------------------------ distributed


def dist_barrier(world):
    D.barrier(world)


def dist_max(v, world, device):
    return D.max_over_ranks(v, world, device)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decoder", choices=sorted(workloads.PRESETS) + ["decoder"],
                    help="'decoder' (default): a whole Qwen3-8B-shaped decoder layer's four "
                         "solves; or a single layer preset")
    ap.add_argument("--bits", type=int, default=0, help="decoder workload: W2/W3/W4 (default 3)")
    ap.add_argument("--solve", default="", choices=["", "qkv", "o", "gate_up", "down"],
                    help="decoder workload: keep only this one of the four solves "
                         "(profiling captures only)")
    ap.add_argument("--no-scaling", action="store_true",
                    help="Sigma = I: the unscaled ablation (objective comparison)")
    ap.add_argument("--rescale-dual", action="store_true",
                    help="variant: V~ *= rho_t / rho_{t+1} after each iteration")
    ap.add_argument("--fit-on-w", action="store_true",
                    help="variant: refresh the grid from Sigma W~ instead of Sigma (W~ + V~)")
    ap.add_argument("--shard", action="store_true",
                    help="split ONE layer over the ranks (tokens and output rows; H all-reduced)")
    ap.add_argument("--grid", default="lsq", choices=["lsq", "minmax", "mse", "frozen"])
    ap.add_argument("--split", default="auto", choices=["auto", "f16", "mixed", "3xtf32"],
                    help="split precision of the eigenbasis GEMMs (auto: f16 from d_in 2048)")
    ap.add_argument("--schedule", default="fused", choices=["fused", "per_gemm"],
                    help="fused: GEMM 1 and GEMM 2 of all iterations in one launch; "
                         "per_gemm: two launches per iteration")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the calibration token count n (profiling captures only; "
                         "the eigenbasis GEMMs do not depend on n)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stream-kernels", action="store_true",
                    help="skip the stand-alone projection / pack bandwidth measurement")
    ap.add_argument("--no-extra", action="store_true",
                    help="decoder workload: skip the q_proj and min/max extra keys")
    ap.add_argument("--no-eigh-overlap", action="store_true",
                    help="decoder workload: skip the eigh-overlap measurement")
    ap.add_argument("--cpu-full", action="store_true",
                    help="--impl reference on a layer preset: the oracle's whole solve, "
                         "no extrapolation")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="--impl reference: limit the BLAS threads (0: all)")
    args = ap.parse_args()
    rank, world, local = D.world()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        runner = run_decoder if args.workload == "decoder" else (run_sharded if args.shard else run_ours)
        line = runner(args, rank, world, device)
        if line:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
