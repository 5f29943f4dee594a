#!/usr/bin/env python
"""Benchmark of the ADMM-Q layer solve on B200.

One step = the hot path of one layer solve on device-resident inputs:
  Gram X^T X (tcgen05, bf16 -> fp32)  ->  damping + diagonal scaling  ->
  C0' GEMM + RTN start  ->  T ADMM iterations (GEMM 1 + GEMM 2 with the fused
  projection / dual update)  ->  residuals + objective  ->  b-bit packing.
The one-time eigendecomposition (cuSOLVER, float64) is outside the step: it
runs during warm-up, is timed on its own and reported as `eigh_s`.

Multi-GPU: layers are independent problems, so every rank solves its own
layer (seed = rank) with no collective in the data path ("scaling": "weak").

    python bench.py [--gpus N --steps K --warmup W --workload q_proj --grid minmax]
    python bench.py --impl reference   # the float64 CPU oracle on a bounded sample
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


def source_hash():
    """Short hash of the CUDA sources (matches the ncu captures in profiles/)."""
    import hashlib
    csrc = os.path.join(ROOT, "post_weight_quantization_10_b200", "csrc")
    per = [hashlib.sha1(open(os.path.join(csrc, f), "rb").read()).hexdigest() + "  " + f
           for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh"))]
    return hashlib.sha1(("\n".join(per) + "\n").encode()).hexdigest()[:12]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` (a preset name) from
    the committed ncu capture, or None when there is no capture of that pair
    or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)[f"{kernel}@{workload}"]
    except (OSError, KeyError, ValueError):
        return None
    return t["dram_bytes_per_launch"] if t["source_hash"] == source_hash() else None


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
        self.X = workloads.make_activations(p, seed=seed, device=device)
        self.W = workloads.make_weights(p, seed=seed, device=device, dtype=torch.bfloat16)
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
        """One layer solve; X / W default to the run's device-resident inputs."""
        A, p = self.A, self.p
        X = self.X if X is None else X
        W = self.W if W is None else W
        mark = (lambda k: ev[k].record()) if ev else (lambda k: None)
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


def run_decoder(args, rank, world, device):
    """One Qwen3-8B-shaped decoder layer per rank: its four solves (q/k/v and
    gate/up stacked on their shared inputs), each timed like the single-layer
    step; the value is the layer's solve time (sum over the four)."""
    from post_weight_quantization_10_b200 import admmq as A
    A.lib()
    bits = args.bits or 3
    solves = []
    n0 = A.launch_count()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for label, p, seed in workloads.decoder_layer(bits):
        if args.tokens:
            p = workloads.scaled(p, args.tokens, p.d_in, p.d_out)
        run = LayerRun(A, p, args.grid, seed=seed + 1000 * rank, device=device, split=args.split,
                       schedule=args.schedule)
        eigh_s = run.setup_eigh()
        for _ in range(args.warmup):
            run.step()
        torch.cuda.synchronize()
        dist_barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        clocks.begin()
        a.record()
        for _ in range(args.steps):
            run.step()
        b.record()
        torch.cuda.synchronize()
        clocks.end()
        ms = dist_max(a.elapsed_time(b), world, device) / args.steps
        obj = objective_report(A, run)
        solves.append({"solve": label, "d_in": p.d_in, "d_out": p.d_out, "bits": p.bits,
                       "iters": p.iters, "s": ms / 1e3, "eigh_s": eigh_s, "split": run.s.split,
                       "iters_per_s": p.iters / (ms / 1e3), "objective": obj})
        del run
        torch.cuda.empty_cache()
    clk = clocks.stop()
    if rank != 0:
        return None
    s_layer = sum(x["s"] for x in solves)
    return {
        "metric": "ADMM-Q decoder-layer solve: s/layer (four solves, eigh separate)",
        "value": s_layer, "unit": "s/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": s_layer * 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None,
        "dtype": " / ".join(sorted({DTYPES[x["split"]] for x in solves})),
        "data": "synthetic (seeded Qwen3-8B-shaped activations and weights; no dataset)",
        "config": {"workload": "Qwen3-8B-shaped decoder layer: qkv 4096->6144, o 4096->4096, "
                               "gate_up 4096->24576, down 12288->4096; W%d g128 T=%d grid=%s"
                               % (bits, solves[0]["iters"], args.grid),
                   "parallelism": f"independent decoder layers x{world}",
                   "l2": "inputs larger than L2"},
        "s_per_layer_with_eigh": s_layer + sum(x["eigh_s"] for x in solves),
        "solves": solves,
        "gpu_launches": A.launch_count() - n0,
        "clocks": clk,
    }


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
    t_start.record()
    for k in range(args.steps):
        run.step(evs[k])
    t_end.record()
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
        e2e = run_e2e(A, run, args, world, device)

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
    # Tensor work per fp32-accurate product, in bf16-MMA units (dense tf32 runs
    # at half the bf16 rate, nominal 1.1 vs 2.25 PFLOP/s): 3xTF32 = three tf32
    # MMAs = 6; fp16 x3 = three full-rate fp16 MMAs = 3; mixed split = one
    # tf32 MMA (2) + one bf16 MMA over the doubled
    # K of the correction rows (2) = 4.  Peak = bf16 peak / that.
    split = run.s.split
    per_product = {"mixed": 4.0, "3xtf32": 6.0, "f16": 3.0}[split]
    peak_split = pk["bf16_sust"] / per_product
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
        line["cpu_baseline"] = cpu_baseline(p, args.grid)
    return line


def stream_kernels(A, grid, device, reps=10):
    """HBM-bound kernels timed on their own, on buffers larger than L2: the
    standalone projection (the fused epilogue's float32 arithmetic reading W~
    from memory) and the b-bit pack.  Algorithmic bytes per element: W~ 4,
    V 4 + 4, codes 1 + 1, P planes 8 (projection); codes 1 + b/8 (pack)."""
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
    phi = torch.empty((m, d), device=device)
    plo = torch.empty((m, 2 * d), dtype=torch.int16, device=device)  # bf16 correction rows
    resid = torch.zeros(2, dtype=torch.float64, device=device)
    big = torch.randint(0, L + 1, (4 * m, d), generator=gen, device=device, dtype=torch.uint8)
    packed = torch.empty((4 * m, d * bits // 32), dtype=torch.int32, device=device)
    out = {}
    for name, fn, nbytes, shape in (
            ("project", lambda: A.project(wt, V, sig, rsig, hd, bits, g, grid, codes, scale, zero,
                                          phi, plo, resid=resid), 22.0 * m * d, [m, d]),
            ("pack", lambda: A.pack(big, bits, out=packed), (1 + bits / 8) * 4 * m * d, [4 * m, d])):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"shape": shape, "bits": bits, "alg_bytes": nbytes, "ms": ms, "gbs": gbs,
                     "frac_hbm": gbs / pk["hbm"], "traffic": measured_traffic(name, "stream")}
    del wt, V, codes, phi, plo, big, packed
    torch.cuda.empty_cache()
    return out


def run_e2e(A, run, args, world, device):
    """The step through the public API from pinned host buffers: every step
    copies its X and W_hat to the device and reads codes, packed words, grid
    and objective back.  The next step's inputs are copied on a second stream
    while the current step runs (pipeline.InputPipeline); the first copy is
    not overlapped."""
    from post_weight_quantization_10_b200.pipeline import InputPipeline
    p = run.p
    Xh = torch.empty(run.X.shape, dtype=run.X.dtype, pin_memory=True)
    Xh.copy_(run.X)
    Wh = torch.empty(run.W.shape, dtype=run.W.dtype, pin_memory=True)
    Wh.copy_(run.W)
    codes_h = torch.empty(run.s.codes.shape, dtype=torch.uint8, pin_memory=True)
    packed_h = torch.empty(run.packed.shape, dtype=torch.int32, pin_memory=True)
    scale_h = torch.empty(run.s.scale.shape, dtype=torch.float32, pin_memory=True)
    zero_h = torch.empty_like(scale_h, pin_memory=True)
    obj_h = torch.empty(1, dtype=torch.float64, pin_memory=True)
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (codes_h, packed_h, scale_h, zero_h, obj_h))
    pipe = InputPipeline([Xh, Wh], device)

    def steps(k):
        slot = pipe.prefetch([Xh, Wh])
        for i in range(k):
            X, W = pipe.acquire(slot)
            nxt = pipe.prefetch([Xh, Wh]) if i + 1 < k else None
            run.step(X=X, W=W)
            pipe.release(slot)
            codes_h.copy_(run.s.codes, non_blocking=True)
            packed_h.copy_(run.packed, non_blocking=True)
            scale_h.copy_(run.s.scale, non_blocking=True)
            zero_h.copy_(run.s.zero, non_blocking=True)
            obj_h.copy_(run.s.objective, non_blocking=True)
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
    run.s.check()
    ms = dist_max(a.elapsed_time(b), world, device)
    return {"value": p.iters * args.steps * world / (ms / 1e3), "unit": "iters/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "s_per_layer": ms / 1e3 / args.steps,
            "overlap": "each step's inputs are copied on a second stream during the previous "
                       "step (the first copy is not overlapped)"}


# --------------------------------------------------- CPU oracle (baseline)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 0) for i in info), default=None)
    except Exception:
        return None


def cpu_sample(p, grid, seed=0):
    """Time the float64 oracle on a bounded sample of the layer: the Gram of
    8192 tokens and one ADMM iteration (W-update, projection, dual update) at
    the full layer size; extrapolate to the step (n tokens, T iterations)."""
    from oracle import admmq_oracle as O
    rng = np.random.default_rng(seed)
    d, m = p.d_in, p.d_out
    ns = min(8192, p.n)
    Xs = rng.standard_normal((ns, d)).astype(np.float32)
    t0 = time.perf_counter()
    O.gram(Xs)
    t_gram = (time.perf_counter() - t0) * (p.n / ns)
    Q = rng.standard_normal((d, d)) / np.sqrt(d)
    lam = np.abs(rng.standard_normal(d)) + 0.1
    B = rng.standard_normal((d, m)) * 0.02
    Dt = rng.standard_normal((d, m)) * 0.02
    Vt = rng.standard_normal((d, m)) * 0.002
    sigma = np.abs(rng.standard_normal(d)) * 0.01 + 0.01
    hdiag = (1.0 / sigma ** 2).astype(np.float32)
    s_prev = np.full((d // p.group, m), 0.01, np.float32)
    z_prev = np.full((d // p.group, m), 3.0, np.float32)
    t0 = time.perf_counter()
    Wt = O.w_update(Q, lam, B, 0.1, Dt, Vt)
    Y = sigma[:, None] * (Wt + Vt)
    _, _, _, D = O.project(Y, p.bits, p.group, grid, hdiag, s_prev, z_prev)
    Vt = Vt + Wt - D / sigma[:, None]
    t_iter = time.perf_counter() - t0
    step_s = t_gram + p.iters * t_iter
    return dict(t_gram=t_gram, t_iter=t_iter, step_s=step_s, iters_per_s=p.iters / step_s,
                sample=f"Gram of {ns} of {p.n} tokens + 1 of {p.iters} ADMM iterations at "
                       f"d_in={d} d_out={m}, extrapolated linearly (eigh excluded, as on the GPU)")


def cpu_baseline(p, grid):
    r = cpu_sample(p, grid)
    return {"value": r["iters_per_s"], "unit": "iters/s", "cores": _blas_threads() or os.cpu_count(),
            "kind": "oracle", "sample": r["sample"], "s_per_layer": r["step_s"]}


def run_reference_decoder(args, world):
    """The oracle on the decoder-layer workload: the bounded sample of each of
    the four solves, summed (seconds per decoder layer)."""
    bits = args.bits or 3
    layers = workloads.decoder_layer(bits)
    for _ in range(args.warmup):
        cpu_sample(layers[0][1], args.grid)
    vals = [sum(cpu_sample(p, args.grid)["step_s"] for _, p, _ in layers) for _ in range(args.steps)]
    value = float(np.mean(vals))
    cores = _blas_threads() or os.cpu_count()
    sample = ("per solve: Gram of 8192 tokens + 1 ADMM iteration at full size, extrapolated "
              "linearly to n and T; summed over the four solves")
    return {"impl": "reference", "metric": "ADMM-Q decoder-layer solve: s/layer (four solves, eigh separate)",
            "value": value, "unit": "s/layer", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": value * 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "Qwen3-8B-shaped decoder layer, W%d g128" % bits},
            "cpu_baseline": {"value": value, "unit": "s/layer", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "s/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    if args.workload == "decoder":
        return run_reference_decoder(args, world)
    p = workloads.PRESETS[args.workload]
    for _ in range(args.warmup):
        cpu_sample(p, args.grid)
    vals = [cpu_sample(p, args.grid) for _ in range(args.steps)]
    step_s = float(np.mean([v["step_s"] for v in vals]))
    value = p.iters / step_s
    cores = _blas_threads() or os.cpu_count()
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "iters/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(p, args.grid)},
            "cpu_baseline": {"value": value, "unit": "iters/s", "cores": cores, "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": value, "unit": "iters/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


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
    ap.add_argument("--workload", default="q_proj", choices=sorted(workloads.PRESETS) + ["decoder"],
                    help="a single layer preset, or 'decoder': a whole decoder layer's four solves")
    ap.add_argument("--bits", type=int, default=0, help="decoder workload: W2/W3/W4 (default 3)")
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
