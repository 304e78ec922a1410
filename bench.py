"""Benchmark of the DP-SGD per-sample clip + sum + noise step on B200.

One step = the whole hot path over one batch: one dp_block_step over the linears of the
workload (Llama-7B-shaped block by default: 7 linears, B=8, T=2048, bf16; the projected
variant passes each linear's P).  It computes the per-sample norms, the clip factors, the
clipped sum and the Gaussian noise of every linear.  The inputs are
seeded synthetic tensors, resident in HBM.  They are larger than the 126 MB L2, and the 7
linears cycle through 2.2 GB, so no L2 flush is needed between steps.

The main line is the 7B block.  The Llama-13B-shaped block (B=4, T=2048) is timed after it in
the same run, with the same steps and warm-up, and reported under "legs" with its own step
time, roofline fractions and per-kernel split.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
Under torchrun every rank runs an independent replica (the step has no cross-GPU exchange).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DP clip+sum+noise tokens/s and TFLOP/s as % of B200 roofline, 1 GPU"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a step's dominant
# kernel, averaged over the step's launches, from one ncu capture of the same command (the
# ncu summaries in profiles/ give the capture).  Each entry records a hash of the code that
# defines that kernel (comments and blank space excluded); when the code changes, the figure
# no longer describes it and bench.py reports traffic as null.
KERNEL_SOURCES = ("sample_gradient_clipping_b200/csrc/ptx.cuh",
                  "sample_gradient_clipping_b200/csrc/umma_gemm.cuh",
                  "sample_gradient_clipping_b200/csrc/umma_gemm_2sm.cuh")
# (workload, kernel) -> (bytes per launch, source hash)
MEASURED_TRAFFIC = {
    ("llama7b_block", "umma_explicit_store"): (895072658, "f293da536260e71b"),
    ("llama13b_block", "umma_explicit_store"): (683888274, "f293da536260e71b"),
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# A timed region at least this long runs under the sustained (power-capped) clock; a shorter
# one is compared with the burst peak.
SUSTAINED_REGION_S = 2.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama7b_block")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="under torchrun: each rank holds its own batch of the workload's size and "
                         "the ranks run one sample-sharded step (NCCL all-reduce of every linear's "
                         "sum, noise added once); default: independent replicas")
    ap.add_argument("--graph", action="store_true",
                    help="replay one CUDA graph per step; the step number lives in device memory and "
                         "the graph advances it")
    ap.add_argument("--no-non-dp", action="store_true",
                    help="skip the non-private comparison (plain bf16 weight-gradient GEMMs)")
    ap.add_argument("--method", default="auto", choices=["auto", "ghost", "explicit", "once"])
    ap.add_argument("--linears", default="", help="comma-separated subset of the workload's linears")
    ap.add_argument("--sigma", type=float, default=None, help="noise multiplier (default: the workload's)")
    ap.add_argument("--also", default="auto",
                    help="comma-separated workloads timed after the main one in the same run and "
                         "reported under 'legs' (default beside the Llama-7B block: the Llama-13B "
                         "block, GPT-2 MLP up and the projected RoBERTa block; 'none' for none)")
    ap.add_argument("--clip", default="per_layer", choices=["per_layer", "flat"],
                    help="per-layer bounds C_l, or one flat bound sqrt(L) * C_l for the whole block")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_model(w):
    """Algorithmic flops and bytes of one step (per-linear sums; X counted per linear)."""
    e = 2 if w.dtype == "bf16" else 4
    N = w.tokens
    flops = byts = 0.0
    x_shared_bytes = 0.0
    seen = set()
    per_linear = []
    for lin in w.linears:
        m, n, r = lin.d_in, lin.d_out, w.r
        if r:
            f = 2.0 * N * n * r + 2.0 * N * m * r
            b = N * m * e + N * n * e + m * r * 4 + n * r * e
        else:
            f = 2.0 * N * m * n
            b = N * m * e + N * n * e + m * n * 4
        flops += f
        byts += b
        x_shared_bytes += b - (N * m * e if lin.x_key in seen else 0)
        seen.add(lin.x_key)
        per_linear.append((lin, f, b))
    return flops, byts, x_shared_bytes, per_linear


def kernel_source_hash():
    """Hash of the dominant kernel's code: its sources with comments and blank space removed,
    so that a comment edit does not void a measurement of unchanged code."""
    import hashlib
    import re

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload, kernel):
    entry = MEASURED_TRAFFIC.get((workload, kernel))
    if entry is None or entry[1] != kernel_source_hash():
        return None
    return entry[0]


def max_over_ranks(value, device, world):
    """The largest of every rank's value (ranks time their own replica; the job is as slow as
    its slowest rank).  Every rank must call it at the same point."""
    if world <= 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_second(tokens_per_replica, world, ms_per_step):
    """Whole-job throughput of `world` replicas that each process `tokens_per_replica` per step."""
    return tokens_per_replica * world / (ms_per_step / 1e3)


def reduce_bytes(w):
    """Bytes of the clipped-sum reduce over stored per-sample tiles: B bf16 reads + one fp32 write."""
    return sum(w.B * l.d_in * (w.r or l.d_out) * 2.0 + l.d_in * (w.r or l.d_out) * 4.0 for l in w.linears)


def ghost_flops(w):
    """Executed flops of the ghost-norm Gram tiles (upper-triangular 128-token tile pairs)."""
    tt = math.ceil(w.T / 128)
    pairs = tt * (tt + 1) // 2
    return sum(w.B * pairs * 2.0 * 128 * 128 * (lin.d_in + (w.r or lin.d_out)) for lin in w.linears)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms during the timed region.

    start() returns once the first sample has arrived, so the sampler is live when timing
    begins; stop() waits for one sample taken after the region, so a region shorter than the
    sampling interval still has a sample on each side of it.
    """

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.reader = None
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            target = str(device_index)
        self.target = target

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line))

    def start(self):
        import threading

        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        deadline = time.monotonic() + 5.0
        while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return None
        t_stop = time.monotonic()
        deadline = t_stop + 1.0
        while time.monotonic() < deadline and not any(t > t_stop for t, _ in self.lines):
            time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.reader is not None:
            self.reader.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- reference arm

def oracle_block_sample(w, data, linears, sample=0):
    """The fp64 oracle on one sample of the given linears; returns (seconds, block-equiv tokens)."""
    import numpy as np

    import oracle
    from sample_gradient_clipping_b200 import inputs

    total_mn = sum(l.d_in * (w.r or l.d_out) for l in w.linears)
    t0 = time.perf_counter()
    tokens = 0.0
    for lin in linears:
        X = inputs.as_f64(data["X"][lin.x_key][sample:sample + 1])
        dY = inputs.as_f64(data["dY"][lin.name][sample:sample + 1])
        P = None
        if w.r:
            P = oracle.round_to(w.dtype, oracle.projection(lin.d_out, w.r, w.seed, lin.layer_id))
        oracle.linear_step(X, dY, w.C, w.sigma, w.seed, w.step, lin.layer_id, P)
        tokens += w.T * lin.d_in * (w.r or lin.d_out) / total_mn
    del np
    return time.perf_counter() - t0, tokens


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        return max(i.get("num_threads", 1) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w, rank):
    if rank != 0:
        return 0
    from sample_gradient_clipping_b200 import inputs

    data = inputs.generate(w)
    lin_cycle = list(w.linears)
    for s in range(args.warmup):
        oracle_block_sample(w, data, [lin_cycle[s % len(lin_cycle)]])
    secs = toks = 0.0
    for s in range(args.steps):
        dt, tk = oracle_block_sample(w, data, [lin_cycle[(args.warmup + s) % len(lin_cycle)]])
        secs += dt
        toks += tk
    value = toks / secs
    cores = blas_threads()
    sample = (f"each step: the fp64 oracle (norms, clip, sum, noise) on sample 0 ({w.T} tokens) of "
              f"one linear, cycling through the {len(w.linears)} linears; tokens counted as the "
              f"linear's share d_in*d_out of the block")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "linears": len(w.linears),
                   "description": w.description},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- our arm

class Prepared:
    """Device tensors and the step function of one workload (one dp_block_step per step)."""


def prepare(args, w, rank, world, dev, stream, shard):
    import torch

    from sample_gradient_clipping_b200 import _lib, inputs

    ctx = Prepared()
    # Sharded: every rank draws its own samples (the noise seed stays the workload's).
    ctx.data = inputs.generate(dataclasses.replace(w, seed=w.seed + 7919 * rank) if shard else w)
    ctx.X = {k: v.to(dev) for k, v in ctx.data["X"].items()}
    ctx.dY = {k: v.to(dev) for k, v in ctx.data["dY"].items()}
    r = w.r
    ctx.G = {l.name: torch.empty(l.d_in, r or l.d_out, dtype=torch.float32, device=dev) for l in w.linears}
    ctx.norms = {l.name: torch.empty(w.B, dtype=torch.float32, device=dev) for l in w.linears}
    # The projection depends on (seed, layer) only, not on the step: it is generated once per
    # linear, as a training loop would, and passed to every step.
    ctx.P = {l.name: _lib.dp_projection_matrix(torch.empty(l.d_out, r, dtype=ctx.X[l.x_key].dtype, device=dev),
                                               w.seed, l.layer_id, stream=stream) for l in w.linears} if r else {}
    flat_C = w.C * math.sqrt(len(w.linears))
    block = [{"X": ctx.X[l.x_key], "dY": ctx.dY[l.name], "layer_id": l.layer_id, "C": w.C, "G_out": ctx.G[l.name],
              "norms_out": ctx.norms[l.name], **({"P": ctx.P[l.name]} if r else {})} for l in w.linears]
    # One block call per step (per-layer or flat clipping; projected layers carry their P).
    if shard and r:
        raise SystemExit("--shard runs unprojected workloads")
    arr = (_lib.DpLayer * len(block))(*[
        _lib.DpLayer(b["X"].data_ptr(), b["dY"].data_ptr(), b["X"].shape[2], b["dY"].shape[2],
                     b["layer_id"], b["C"], b["G_out"].data_ptr(), b["norms_out"].data_ptr(),
                     b["P"].data_ptr() if "P" in b else None, r)
        for b in block])
    ws_bytes = _lib.lib().dp_block_workspace_size(arr, len(block), w.B, w.T,
                                                  _lib.DP_BF16 if w.dtype == "bf16" else _lib.DP_F32,
                                                  _lib.CLIP_MODES[args.clip], _lib.METHODS[args.method])
    ctx.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flat_norms = torch.empty(w.B, dtype=torch.float32, device=dev)
    if shard:
        from sample_gradient_clipping_b200 import sharded

        shard_ops = sharded.LibraryOps(args.method)

    def step(k):
        k = w.step + k if isinstance(k, int) else k   # a number, or the device step counter
        if shard:
            sharded.sharded_step(block, w.sigma, w.seed, k, mode=args.clip, C=flat_C, ops=shard_ops)
            return
        _lib.dp_block_step(block, mode=args.clip, C=flat_C if args.clip == "flat" else w.C, sigma=w.sigma,
                           seed=w.seed, step=k, method=args.method,
                           flat_norms_out=flat_norms if args.clip == "flat" else None, workspace=ctx.ws,
                           stream=stream)

    ctx.step = step
    return ctx


def measure(args, w, ctx, world, dev, stream, local):
    """Warm-up, then K timed steps (CUDA events on the launching stream, barrier and
    synchronize on both sides), then a second pass over the same steps with an event pair
    around every launch for the per-kernel split.  Returns the measurements of this rank."""
    import torch

    from sample_gradient_clipping_b200 import _lib

    step = ctx.step
    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(dev)
    if _lib.dp_workspace_status(ctx.ws, stream) != _lib.DP_OK:
        raise RuntimeError("an in-kernel wait timed out during warm-up")

    graph, graph_launches = None, 0
    if args.graph:
        # The step counter starts where the ordinary steps of the timed pass would, and the
        # graph increments it after each step, so every replay draws the next step's noise.
        step_dev = torch.full((1,), w.step + args.warmup, dtype=torch.int64, device=dev)
        graph = torch.cuda.CUDAGraph()
        l0 = _lib.kernel_launches()
        with torch.cuda.graph(graph, stream=stream):
            step(step_dev)
            step_dev.add_(1)
        graph_launches = _lib.kernel_launches() - l0
        graph.replay()
        torch.cuda.synchronize(dev)
        step_dev.fill_(w.step + args.warmup)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = _lib.kernel_launches()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for k in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step(args.warmup + k)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    # Graph replays launch the kernels the capture recorded; the host counter saw them once.
    launches = graph_launches * args.steps if graph is not None else _lib.kernel_launches() - launches0
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    # Per-kernel device times come from a second pass over the same steps with a CUDA event
    # pair around every launch.  The events cost a few microseconds a launch, which is noise
    # on the Llama blocks but a large share of the small workloads' steps, so they stay out of
    # the pass that gives `value`.
    _lib.profiling_enable(True)
    _lib.profiling_collect()
    pv0, pv1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pv0.record(stream)
    for k in range(args.steps):
        step(args.warmup + k)
    pv1.record(stream)
    torch.cuda.synchronize(dev)
    prof = _lib.profiling_collect()
    _lib.profiling_enable(False)
    profiled_ms = pv0.elapsed_time(pv1) / args.steps
    if _lib.dp_workspace_status(ctx.ws, stream) != _lib.DP_OK:
        raise RuntimeError("an in-kernel wait timed out during the timed steps")
    if graph is not None:
        del graph
    return {"ms": max_over_ranks(ms, dev, world), "launches": launches, "clocks": clocks, "prof": prof,
            "profiled_ms": profiled_ms}


def roofline_report(args, w, meas, world):
    """tflops_alg, step_roofline, the dominant kernel's roofline and the per-kernel split.

    A tensor-bound kernel is divided by the measured burst bf16 peak unless the timed region
    itself lasts seconds (then the sustained, power-capped figure applies); both fractions
    are printed, each labelled."""
    pk, pk_kind = peaks()
    flops, byts, xbytes, per_linear = workload_model(w)
    ms = meas["ms"]
    roof_t_burst = max(flops / (pk["bf16_tflops"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    roof_t_sust = max(flops / (pk["bf16_tflops_sustained"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    step_s = ms / 1e3
    region_s = step_s * args.steps
    kinds = dict(meas["prof"])
    dominant = max(kinds, key=lambda k: kinds[k][0]) if kinds else None
    roofline = None
    if dominant:
        d_ms, d_n = kinds[dominant]
        if dominant == "umma_clipsum":
            work, unit, bound = flops * args.steps, "TFLOP/s", "tensor"
        elif dominant == "umma_ghost_norm":
            work, unit, bound = ghost_flops(w) * args.steps, "TFLOP/s", "tensor"
        elif dominant in ("umma_explicit_norm", "umma_explicit_store"):
            work, unit, bound = flops * args.steps, "TFLOP/s", "tensor"
        elif dominant == "clip_reduce":
            work, unit, bound = reduce_bytes(w) * args.steps, "GB/s", "hbm"
        else:
            work, unit, bound = None, None, None
        if work is not None:
            if unit == "GB/s":
                achieved = work / (d_ms / 1e3) / 1e9
                peak, peak_kind = pk["hbm_gbs"], f"{pk_kind} HBM copy bandwidth"
                extra = {}
            else:
                achieved = work / (d_ms / 1e3) / 1e12
                long_region = region_s >= SUSTAINED_REGION_S
                burst, sust = pk["bf16_tflops"], pk["bf16_tflops_sustained"]
                peak = sust if long_region else burst
                peak_kind = (f"{pk_kind} sustained bf16 (timed region {region_s:.2f} s, seconds long)" if long_region
                             else f"{pk_kind} burst bf16 (timed region {region_s:.2f} s, under "
                                  f"{SUSTAINED_REGION_S:g} s)")
                extra = {"frac_of_burst": achieved / burst, "peak_burst": burst,
                         "frac_of_sustained": achieved / sust, "peak_sustained": sust}
            roofline = {"bound": bound, "kernel": dominant, "achieved": achieved, "peak": peak,
                        "unit": unit, "frac": achieved / peak, **extra,
                        "traffic": measured_traffic(w.name, dominant),
                        "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                        "peak_kind": peak_kind,
                        "launches": d_n // args.steps, "avg_launch_ms": d_ms / d_n,
                        "share_of_step": d_ms / (meas["profiled_ms"] * args.steps)}
    return {
        "tflops_alg": flops * world / step_s / 1e12,
        "step_roofline": {"frac_of_burst": roof_t_burst / step_s, "frac_of_sustained": roof_t_sust / step_s,
                          "roofline_ms_burst": roof_t_burst * 1e3, "roofline_ms_sustained": roof_t_sust * 1e3,
                          "peaks": pk_kind, "bytes_alg": byts, "bytes_alg_x_shared": xbytes, "flops_alg": flops,
                          "executed_ghost_flops": ghost_flops(w)},
        "roofline": roofline,
        "kernels": {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
                    for k, v in sorted(kinds.items(), key=lambda kv: -kv[1][0])},
        "kernel_timing": {"how": "CUDA events around every launch, in a second pass over the same steps"
                                 + (" launched from the host (no graph)" if args.graph else ""),
                          "ms_per_step_with_events": meas["profiled_ms"]},
    }


def workload_config(args, w, world, shard):
    return {"workload": w.name, "B": w.B, "T": w.T, "linears": len(w.linears),
            "method": args.method, "clip": args.clip, "l2": "inputs larger than L2 (no flush)",
            "launch": ("one CUDA graph replay per step (device-resident step counter)" if args.graph
                       else "library calls from the host every step"),
            "parallelism": (f"dp{world}: samples sharded, one NCCL all-reduce per linear, noise "
                            "added once" if shard else "replicas" if world > 1 else "1 GPU"),
            **({"projection": f"P [d_out, {w.r}] generated once per linear before timing "
                              "(it depends on seed and layer only)"} if w.r else {}),
            "description": w.description}


def extra_legs(args, w, shard):
    """Workloads timed after the main one in the same run (same steps and warm-up)."""
    if shard or args.also == "none":
        return []
    if args.also == "auto":
        return ["llama13b_block", "gpt2_mlp_up", "roberta_large_projected"] if w.name == "llama7b_block" else []
    return [n for n in args.also.split(",") if n and n != w.name]


def run_ours(args, w, rank, world):
    import torch

    from sample_gradient_clipping_b200 import _lib, inputs

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    _lib.lib()
    shard = args.shard and world > 1
    if shard and args.graph:
        raise SystemExit("--shard runs without --graph")
    # A graph is captured on a side stream; everything then runs on that stream.
    stream = torch.cuda.Stream(dev) if args.graph else torch.cuda.current_stream(dev)
    torch.cuda.set_stream(stream)
    ctx = prepare(args, w, rank, world, dev, stream, shard)
    meas = measure(args, w, ctx, world, dev, stream, local)
    ms = meas["ms"]

    # ---- the non-private step of the same shapes, for FlashDP's "share of non-DP throughput"
    non_dp = None
    if not args.no_non_dp and w.r == 0 and w.dtype == "bf16":
        non_dp = run_non_dp(args, w, ctx.X, ctx.dY, dev, stream, torch, world, ms)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and shard:
        e2e = {"unavailable": "the end-to-end leg times the one-GPU call; run it without --shard"}
    elif not args.no_e2e:
        e2e = run_e2e(args, w, ctx.data, dev, stream, w.r, ctx.P, _lib, torch, world)

    data = ctx.data
    del ctx
    torch.cuda.empty_cache()

    # ---- further workloads in the same run (the Llama-13B block and the two small
    # configurations beside the 7B one)
    legs = {}
    for name in extra_legs(args, w, shard):
        lw = inputs.WORKLOADS[name]
        lctx = prepare(args, lw, rank, world, dev, stream, shard)
        lmeas = measure(args, lw, lctx, world, dev, stream, local)
        lnon = None
        if not args.no_non_dp and lw.r == 0 and lw.dtype == "bf16":
            lnon = run_non_dp(args, lw, lctx.X, lctx.dY, dev, stream, torch, world, lmeas["ms"])
        legs[name] = {"value": job_tokens_per_second(lw.tokens, world, lmeas["ms"]), "unit": "tokens/s",
                      "ms_per_step": lmeas["ms"], "config": workload_config(args, lw, world, shard),
                      **roofline_report(args, lw, lmeas, world), "gpu_launches": lmeas["launches"],
                      "clocks": lmeas["clocks"], "non_dp": lnon}
        del lctx
        torch.cuda.empty_cache()

    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": job_tokens_per_second(w.tokens, world, ms), "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(args, w, world, shard),
        **roofline_report(args, w, meas, world),
        "gpu_launches": meas["launches"],
        "clocks": meas["clocks"],
        "e2e": e2e,
        "non_dp": non_dp,
    }
    if legs:
        line["legs"] = legs
    if world == 1 and not args.no_cpu_baseline:
        secs, toks = oracle_block_sample(w, data, list(w.linears))
        line["cpu_baseline"] = {
            "value": toks / secs, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"sample 0 ({w.T} tokens) through all {len(w.linears)} linears with the fp64 "
                      f"oracle (norms, clip, sum, full noise), {secs:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


def run_non_dp(args, w, X, dY, dev, stream, torch, world, dp_ms):
    """Plain weight gradients X^T dY of every linear, bf16 in, fp32 out, by cuBLAS (torch.mm).

    This is what a non-private step computes for these linears: no per-sample norms, no
    clipping, no noise.  It is a comparison only; nothing of it is on the library's path.
    """
    outs = {l.name: torch.empty(l.d_in, l.d_out, dtype=torch.float32, device=dev) for l in w.linears}
    Xf = {k: v.view(-1, v.shape[-1]) for k, v in X.items()}
    dYf = {k: v.view(-1, v.shape[-1]) for k, v in dY.items()}

    def step():
        for l in w.linears:
            torch.mm(Xf[l.x_key].t(), dYf[l.name], out_dtype=torch.float32, out=outs[l.name])

    try:
        step()
    except (RuntimeError, NotImplementedError, TypeError) as e:  # no fp32-output bf16 mm here
        return {"unavailable": f"torch.mm with out_dtype=float32: {type(e).__name__}"}

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
        torch.cuda.synchronize(dev)
        steps = max(5, min(args.steps, 50))
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, dev, world)
    return {"what": "X^T dY per linear by cuBLAS (torch.mm, bf16 in, fp32 out); no norms, clipping or noise",
            "ms_per_step": ms, "steps": steps, "tokens_per_s": job_tokens_per_second(w.tokens, world, ms),
            "dp_share_of_non_dp_throughput": ms / dp_ms}


def run_e2e(args, w, data, dev, stream, r, P, _lib, torch, world):
    """Same step through the public API from pinned host buffers, copies inside the timing.

    Three streams: host->device copies of each linear's inputs, dp_linear_step on the compute
    stream, and device->host copies of its outputs.  They overlap layer by layer: linear l+1
    uploads while l computes and l-1 downloads (PCIe is full duplex).  CUDA events order
    every dependency, including the reuse of a device buffer by the next step.
    """
    hX = {k: v.pin_memory() for k, v in data["X"].items()}
    hdY = {k: v.pin_memory() for k, v in data["dY"].items()}
    # One linear at a time through dp_linear_step: its own workspace, sized for the largest.
    ws = torch.empty(max(_lib.workspace_size(w.B, w.T, l.d_in, l.d_out, r,
                                             _lib.DP_BF16 if w.dtype == "bf16" else _lib.DP_F32, args.method)
                         for l in w.linears), dtype=torch.uint8, device=dev)
    dX = {k: torch.empty_like(v, device=dev) for k, v in hX.items()}
    ddY = {k: torch.empty_like(v, device=dev) for k, v in hdY.items()}
    G = {l.name: torch.empty(l.d_in, r or l.d_out, dtype=torch.float32, device=dev) for l in w.linears}
    n = {l.name: torch.empty(w.B, dtype=torch.float32, device=dev) for l in w.linears}
    hG = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in G.items()}
    hn = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in n.items()}
    bi = sum(v.numel() * v.element_size() for v in hX.values()) + \
        sum(v.numel() * v.element_size() for v in hdY.values())
    bo = sum(v.numel() * v.element_size() for v in hG.values()) + \
        sum(v.numel() * v.element_size() for v in hn.values())
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    # last use of each device buffer (compute of the previous step) and of each output
    x_free = {k: None for k in dX}
    dy_free = {k: None for k in ddY}
    out_free = {k: None for k in G}

    def step(k):
        loaded = {}
        for l in w.linears:
            with torch.cuda.stream(up):
                if l.x_key not in loaded:
                    if x_free[l.x_key] is not None:
                        up.wait_event(x_free[l.x_key])
                    dX[l.x_key].copy_(hX[l.x_key], non_blocking=True)
                    e = ev(); e.record(up); loaded[l.x_key] = e
                if dy_free[l.name] is not None:
                    up.wait_event(dy_free[l.name])
                ddY[l.name].copy_(hdY[l.name], non_blocking=True)
                dy_ready = ev(); dy_ready.record(up)
            stream.wait_event(loaded[l.x_key])
            stream.wait_event(dy_ready)
            if out_free[l.name] is not None:
                stream.wait_event(out_free[l.name])
            _lib.dp_linear_step(dX[l.x_key], ddY[l.name], w.C, w.sigma, w.seed, w.step + k, l.layer_id,
                                P=P.get(l.name), r=r, method=args.method, norms_out=n[l.name],
                                G_out=G[l.name], workspace=ws, stream=stream)
            done = ev(); done.record(stream)
            x_free[l.x_key] = done
            dy_free[l.name] = done
            with torch.cuda.stream(down):
                down.wait_event(done)
                hG[l.name].copy_(G[l.name], non_blocking=True)
                hn[l.name].copy_(n[l.name], non_blocking=True)
                read = ev(); read.record(down)
                out_free[l.name] = read

    steps = max(1, min(args.steps, 5))
    for k in range(min(args.warmup, 2)):
        step(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    up.wait_event(ev0)
    for k in range(steps):
        step(k)
    down.synchronize()
    stream.wait_stream(down)
    stream.wait_stream(up)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, dev, world)
    return {"value": job_tokens_per_second(w.tokens, world, ms), "unit": "tokens/s", "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "ms_per_step": ms, "steps": steps,
            "result_read_back": "every linear's noisy clipped gradient and per-sample norms",
            "overlap": "uploads, compute and downloads on three streams, layer by layer"}


def main():
    args = parse()
    from sample_gradient_clipping_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    if args.linears:
        keep = args.linears.split(",")
        lins = tuple(l for l in w.linears if l.name in keep)
        if not lins:
            raise SystemExit(f"no linear of {w.name} in {keep}")
        w = dataclasses.replace(w, name=f"{w.name}[{args.linears}]", linears=lins)
    if args.sigma is not None:
        w = dataclasses.replace(w, name=f"{w.name}[sigma={args.sigma:g}]", sigma=args.sigma)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, w, rank)
    if world > 1:
        import torch

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, w, rank, world)
    finally:
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
