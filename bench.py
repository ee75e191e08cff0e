#!/usr/bin/env python
"""Benchmark of the bf16 causal self-attention hot path (forward + backward) on B200.

One step = one forward (attn_fwd) and one backward (attn_bwd's three stages: preprocess, dK/dV with dQ
accumulation, dQ conversion) over one batch of the workload, inputs resident in HBM. The metric is causal
TFLOP/s with the convention fwd = 2*B*H*T^2*D and bwd = 2.5 x fwd, and its fraction of the measured dense
bf16 tensor peak. Launch:

  python bench.py [--gpus 1] [--steps K] [--warmup W] [--workload d20] [--impl ours|reference]
  torchrun --nproc-per-node N bench.py --gpus N ...      (replicas: every rank runs its own batch)

Rank 0 prints one JSON line. ``--impl reference`` times the float64 CPU oracle (the only reference this
path has) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, Workload  # noqa: E402

METRIC = "causal attention fwd+bwd TFLOP/s (bf16, d20 shape) and % of B200 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
KERNEL_SOURCES = ["attn_api.cu", "attn_fwd.cuh", "attn_bwd.cuh", "attn_decode.cuh", "attn_common.cuh", "attn_errors.h",
                  "sm100.cuh"]
PROLOGUE_SOURCES = ["attn_rope.cu"]  # the prologue's kernels and launches are all in this file


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    from workloads import DECODE_WORKLOADS, PROLOGUE_WORKLOADS
    ap.add_argument("--workload", default="d20",
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(PROLOGUE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--sustained-seconds", type=float, default=2.5,
                    help="length of the sustained leg (the same step looped, with its own clock record); 0 skips it")
    return ap.parse_args(argv)


# ------------------------------------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "causal_self_attention_bf16_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, sources=KERNEL_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    ent = d.get(kernel, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash(sources):
        return None
    return ent.get("dram_bytes_per_launch")


def flops(w: Workload):
    """Forward and backward FLOPs of the metric's convention (causal half; a sliding window scales it by the
    fraction of causal pairs inside the window)."""
    return w.fwd_flops, w.bwd_flops


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (identity at world size 1). Works with nccl (device tensor) and gloo (CPU tensor)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return per_rank_units * world / max_seconds


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled in the background during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        text = self.file.read()
        self.file.close()
        os.unlink(self.file.name)
        return summarize_clocks(text)


def summarize_clocks(text: str):
    """Median SM clock, the maximum clock and power, and every throttle reason seen Active, from nvidia-smi's
    `--query-gpu=ClockSampler.FIELDS --format=csv,noheader,nounits` lines. Rows that do not parse (a line cut
    off when the sampler is stopped, "[N/A]" values) are skipped."""
    rows = [r.split(",") for r in text.strip().splitlines() if r.count(",") >= 8]
    sm, smax, power, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        try:
            vals = float(r[1]), float(r[2]), float(r[3])
        except ValueError:
            continue
        sm.append(vals[0])
        smax.append(vals[1])
        power.append(vals[2])
        for name, val in zip(names, r[5:9]):
            if val.strip().lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
            "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------ CPU oracle

def oracle_sample(w: Workload, seconds: float, min_slices: int = 2, max_slices: int = 256):
    """Time the float64 oracle (fwd + bwd) on seeded (b, h) slices of the workload's shape on the host cores.

    Slices are independent problems of identical cost, so TFLOP/s over a sample equals TFLOP/s over the
    whole batch. Returns (TFLOP/s, cores, description, seconds).
    """
    import numpy as np  # noqa: F401
    from threadpoolctl import threadpool_limits

    from oracle import attn_ref
    from workloads import make_inputs

    cores = len(os.sched_getaffinity(0))
    with threadpool_limits(limits=cores):
        probe = make_inputs(w.with_shape(B=1, H=1, Hkv=0, seed=w.seed + 1000))
        t0 = time.perf_counter()
        win = w.window if w.window >= 0 else None
        attn_ref.slice_forward_backward(*probe, 0, 0, w.scale, window=win)
        t1 = time.perf_counter() - t0
        k = int(max(min_slices, min(max_slices, round(seconds / max(t1, 1e-6)))))
        q, kk, v, do = make_inputs(w.with_shape(B=1, H=k, Hkv=1 if w.kv_heads != w.H else 0, seed=w.seed + 1001))
        t0 = time.perf_counter()
        for h in range(k):
            attn_ref.slice_forward_backward(q, kk, v, do, 0, h, w.scale, window=win)
        dt = time.perf_counter() - t0
    f_slice = 3.5 * w.with_shape(B=1, H=1).fwd_flops
    tflops = k * f_slice / dt / 1e12
    desc = (f"{k} (b,h) slices of {w.name} (T={w.T}, D={w.D}), fwd+bwd float64 numpy, "
            f"{dt:.1f} s; equal-cost independent slices, so the rate holds for the full batch of {w.B * w.H}")
    return tflops, cores, desc, dt


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0  # the reference arm runs on rank 0 only
    w = WORKLOADS[args.workload]
    from threadpoolctl import threadpool_limits

    from oracle import attn_ref
    from workloads import make_inputs

    cores = len(os.sched_getaffinity(0))
    slices = 2  # per step: a bounded sample of the workload
    q, k, v, do = make_inputs(w.with_shape(B=1, H=slices, Hkv=1 if w.kv_heads != w.H else 0, seed=w.seed + 2000))
    times = []
    with threadpool_limits(limits=cores):
        for it in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            for h in range(slices):
                attn_ref.slice_forward_backward(q, k, v, do, 0, h, w.scale,
                                                window=w.window if w.window >= 0 else None)
            if it >= args.warmup:
                times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    f_step = slices * 3.5 * w.with_shape(B=1, H=1).fwd_flops
    value = f_step / step / 1e12
    sample = f"{slices} (b,h) slices of {w.name} per step, float64 numpy oracle fwd+bwd"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": dict(workload_config(w), parallelism=f"replicas x{args.gpus} (no collective on the data path)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: Workload):
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.kv_heads, "T": w.T, "D": w.D, "causal": True,
            "window": w.window,
            "scale": "1/sqrt(D)", "recipe": w.recipe,
            "flop_convention": "fwd 2*B*H*T^2*D (with a window: times the fraction of causal pairs inside it), "
                               "bwd 2.5x fwd",
            "l2": "no flush: q,k,v,dO together exceed the 126 MB L2" if 4 * w.B * w.T * w.H * w.D * 2 > 126e6
            else "inputs smaller than L2"}


# ------------------------------------------------------------------------------------------------ GPU arm

def make_device_inputs(w: Workload, device):
    """The workload's seeded inputs (workloads.make_inputs: the same CPU generator and bytes the parity tests
    check), copied to the device."""
    from workloads import make_inputs
    return [t.to(device) for t in make_inputs(w)]


def run_ours(args):
    import torch

    import causal_self_attention_bf16_b200 as attn

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOADS[args.workload]
    lib = attn.load_library()
    B, H, T, D = w.B, w.H, w.T, w.D
    Hkv = w.kv_heads
    window = w.window  # -1: no sliding window
    gqa = Hkv != H or window >= 0  # grouped-query attention (k, v, dk, dv have Hkv heads) or a sliding window
    scale = w.scale
    q, k, v, do = make_device_inputs(w, device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = attn.attn_bwd_workspace_bytes(B, H, T, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream
    bwd_args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws_bytes, B, H, T, D, scale, sh)

    def check(st, name):
        if st != 0:
            raise RuntimeError(f"{name}: {attn._STATUS.get(st, st)} {lib.attn_last_cuda_error().decode()}")

    if not gqa:
        # Four launches, each bracketed by events for the per-kernel roofline.
        names = ["attn_fwd_kernel", "attn_bwd_prep_kernel", "attn_bwd_dkdv_kernel", "attn_bwd_dq_kernel"]
        calls = [lambda: check(lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                            B, H, T, D, scale, sh), "attn_fwd"),
                 lambda: check(lib.attn_bwd_preprocess(*bwd_args), "attn_bwd_preprocess"),
                 lambda: check(lib.attn_bwd_dkdv(*bwd_args), "attn_bwd_dkdv"),
                 lambda: check(lib.attn_bwd_dq_convert(*bwd_args), "attn_bwd_dq_convert")]
    else:
        # General entry points (key/value heads, window): the forward kernel, then the whole backward (its
        # three kernels).
        ex_bwd_args = bwd_args[:11] + (B, H, Hkv, T, D, scale, window, sh)
        names = ["attn_fwd_kernel", "attn_bwd_ex"]
        calls = [lambda: check(lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                               lse.data_ptr(), B, H, Hkv, T, D, scale, window, sh), "attn_fwd_ex"),
                 lambda: check(lib.attn_bwd_ex(*ex_bwd_args), "attn_bwd_ex")]

    def step(ev=None):
        for j, call in enumerate(calls):
            if ev is not None:
                ev[j].record(stream)
            call()
        if ev is not None:
            ev[len(calls)].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    if attn.get_device_error() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(gpu_id)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    time.sleep(0.1)  # let the sampler start before the timed region
    start.record(stream)
    for i in range(args.steps):
        step(events[i])
    end.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    err = attn.get_device_error()
    if err != 0:
        raise RuntimeError(f"a kernel gave up on a bounded wait (error word {err:#x}); no number is reported")
    per = {n: [] for n in names}
    for ev in events:
        for j, n in enumerate(names):
            per[n].append(ev[j].elapsed_time(ev[j + 1]))
    avg = {n: sum(v_) / len(v_) for n, v_ in per.items()}
    max_total_ms = reduce_max(total_ms, world, device)
    ms_step = max_total_ms / args.steps
    f_fwd, f_bwd = flops(w)
    value = aggregate((f_fwd + f_bwd) * args.steps, world, max_total_ms / 1e3) / 1e12

    peaks = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    peak_tf_sus = float(peaks.get("bf16_tflops_sustained", peak_tf))
    hbm = float(peaks["hbm_gbs"])
    n = B * T * H * D
    nkv = B * T * Hkv * D
    kernels = {
        "attn_fwd_kernel": {"bound": "tensor", "unit": "TFLOP/s", "work": f_fwd, "per": 1e12,
                            "alg_bytes": (2 * n + 2 * nkv) * 2 + B * H * T * 4},
        "attn_bwd_prep_kernel": {"bound": "hbm", "unit": "GB/s", "work": 2 * n * 2 + B * H * T * 4 * 3 +
                                 B * H * ((T + 127) // 128 * 128) * 128 * 4, "per": 1e9},
        "attn_bwd_dkdv_kernel": {"bound": "tensor", "unit": "TFLOP/s", "work": f_bwd, "per": 1e12,
                                 "alg_bytes": 7 * n * 2 + B * H * T * 8},
        "attn_bwd_dq_kernel": {"bound": "hbm", "unit": "GB/s", "work": n * 4 + n * 2, "per": 1e9},
        "attn_bwd_ex": {"bound": "tensor", "unit": "TFLOP/s", "work": f_bwd, "per": 1e12},
    }
    kernels = {name: kernels[name] for name in names}
    breakdown = {}
    for name, kinfo in kernels.items():
        t = avg[name] / 1e3
        ach = kinfo["work"] / t / kinfo["per"]
        pk = peak_tf if kinfo["bound"] == "tensor" else hbm
        breakdown[name] = {"avg_ms": avg[name], "share": avg[name] / sum(avg.values()), "achieved": ach,
                           "unit": kinfo["unit"], "frac": ach / pk}
    dom = max(avg, key=avg.get)
    kd = kernels[dom]
    ach = breakdown[dom]["achieved"]
    pk = peak_tf if kd["bound"] == "tensor" else hbm
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": ach, "peak": pk, "unit": kd["unit"],
                "frac": ach / pk, "traffic": recorded_traffic(dom, w.name),
                "peak_source": f"{peaks['source']} ({'bf16_tflops burst' if kd['bound'] == 'tensor' else 'hbm_gbs'})"}
    if kd["bound"] == "tensor":
        roofline["frac_of_sustained_peak"] = ach / peak_tf_sus

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": dict(workload_config(w), parallelism=f"replicas x{world} (no collective on the data path)"),
        "pct_of_peak": 100.0 * (value / world) / peak_tf,
        "fwd_tflops": f_fwd / (avg["attn_fwd_kernel"] / 1e3) / 1e12,
        "bwd_tflops": f_bwd / (sum(avg.values()) - avg["attn_fwd_kernel"]) * 1e3 / 1e12,
        "roofline": roofline, "kernels": breakdown, "gpu_launches": 4 * args.steps, "clocks": clocks,
        "kernel_source_hash": kernel_source_hash(),
    }

    # Sustained leg: the same step back to back for a few seconds, its own clock record, against the sustained
    # (power-capped) GEMM peak. The headline value stays the timed steps above (a burst of args.steps steps).
    if args.sustained_seconds > 0:
        n_sus = max(1, int(math.ceil(args.sustained_seconds * 1e3 / ms_step)))
        sampler = ClockSampler(gpu_id)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)
        sampler.start()
        time.sleep(0.1)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(n_sus):
            step()
        s1.record(stream)
        torch.cuda.synchronize(device)
        sus_clocks = sampler.stop()
        sus_ms = reduce_max(s0.elapsed_time(s1), world, device)
        sus_value = aggregate((f_fwd + f_bwd) * n_sus, world, sus_ms / 1e3) / 1e12
        line["sustained"] = {"value": sus_value, "unit": UNIT, "steps": n_sus, "seconds": sus_ms / 1e3,
                             "ms_per_step": sus_ms / n_sus, "pct_of_sustained_peak": 100.0 * (sus_value / world) /
                             peak_tf_sus, "peak": peak_tf_sus, "clocks": sus_clocks}
        line["gpu_launches_sustained"] = 4 * n_sus  # forward + the backward's three kernels, per step

    # End to end through the public Python API with host buffers: H2D of q, k, v, dO from pinned memory,
    # forward, backward, D2H of o, lse, dq, dk, dv, every step.
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
        ho, hdq = (torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2))
        hdk, hdv = (torch.empty(k.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2))
        hlse = torch.empty((B, H, T), dtype=torch.float32).pin_memory()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            do.copy_(hdo, non_blocking=True)
            win = window if window >= 0 else None
            attn.attn_fwd(q, k, v, scale, o=o, lse=lse, window=win)
            attn.attn_bwd(q, k, v, o, lse, do, scale, dq=dq, dk=dk, dv=dv, workspace=ws, window=win)
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
            hdq.copy_(dq, non_blocking=True)
            hdk.copy_(dk, non_blocking=True)
            hdv.copy_(dv, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(device)
        e_steps = 5
        if world > 1:
            torch.distributed.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = reduce_max(s0.elapsed_time(s1), world, device)
        line["e2e"] = {"value": aggregate((f_fwd + f_bwd) * e_steps, world, e_ms / 1e3) / 1e12, "unit": UNIT,
                       "h2d_bytes_per_step": (2 * n + 2 * nkv) * 2,
                       "d2h_bytes_per_step": (2 * n + 2 * nkv) * 2 + B * H * T * 4,
                       "ms_per_step": e_ms / e_steps}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, cores, desc, _ = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = "KV-cache decode attention HBM GB/s (bf16 cache)"


def decode_bytes(w, lens):
    """Algorithmic bytes of one decode call: the K and V rows some query sees (all valid rows, or with a sliding
    window the last Tq + window of them), q, o and lse."""
    seen = [int(x) if w.window < 0 else min(int(x), w.Tq + w.window) for x in lens]
    kv = sum(seen) * w.Hkv * w.D * 2 * 2
    return kv + 2 * w.B * w.Tq * w.H * w.D * 2 + w.B * w.H * w.Tq * 4


def run_decode(args):
    """Cached decode (forward only): HBM-bound, measured in GB/s of algorithmic bytes against the measured
    copy bandwidth. Inputs (q, caches over 1 GB in all for the d20 workloads) are resident; no L2 flush needed
    when the cache exceeds L2, which the line states."""
    from workloads import DECODE_WORKLOADS, make_decode_inputs
    w = DECODE_WORKLOADS[args.workload]
    rank, world, _ = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        from threadpoolctl import threadpool_limits

        from oracle import attn_ref
        q, kc, vc, lens = make_decode_inputs(w)
        n = min(w.B, 4)
        times = []
        with threadpool_limits(limits=len(os.sched_getaffinity(0))):
            for it in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                attn_ref.decode_forward(q[:n], kc[:n], vc[:n], lens[:n].numpy(), w.scale,
                                        window=w.window if w.window >= 0 else None)
                if it >= args.warmup:
                    times.append(time.perf_counter() - t0)
        sw = dataclasses.replace(w, B=n)
        value = decode_bytes(sw, lens[:n]) / (sum(times) / len(times)) / 1e9
        print(json.dumps({"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
                          "dtype": "f64", "data": "synthetic", "config": {"workload": w.name, "recipe": w.recipe},
                          "cpu_baseline": {"value": value, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
                                           "kind": "oracle", "sample": f"{n} sequences of {w.name} per step"},
                          "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    import torch

    import causal_self_attention_bf16_b200 as attn
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    q, kc, vc, lens = (t.to(device) for t in make_decode_inputs(w))
    o, lse = torch.empty_like(q), torch.empty((w.B, w.H, w.Tq), dtype=torch.float32, device=device)
    lib = attn.load_library()
    ws_bytes = int(lib.attn_decode_workspace_bytes(w.B, w.H, w.Hkv, w.Tq, w.Tk, w.D))
    per_call = int(lib.attn_decode_kernels(w.B, w.H, w.Hkv, w.Tq, w.Tk, w.D, w.window))  # kernels per call
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    sh = torch.cuda.current_stream(device).cuda_stream

    def call():
        st = lib.attn_decode_ex(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), ws.data_ptr(), ws_bytes, w.B, w.H, w.Hkv, w.Tq, w.Tk, w.D, w.scale,
                                w.window, sh)
        if st != 0:
            raise RuntimeError(f"attn_decode: {attn._STATUS.get(st, st)}")

    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize(device)
    # The cache of one call is smaller than L2 for some workloads: a 256 MB buffer is written between calls.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(gpu_id)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    time.sleep(0.1)
    for e0, e1 in ev:
        flush.zero_()
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    if attn.get_device_error() != 0:
        raise RuntimeError("a decode kernel reported an error")
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev) / len(ev), world, device)  # slowest rank
    nbytes = decode_bytes(w, lens.cpu())
    gbs = nbytes / (ms / 1e3) / 1e9
    hbm = float(load_peaks()["hbm_gbs"])
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    print(json.dumps({
        "metric": DECODE_METRIC, "value": gbs * world, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.Hkv, "Tq": w.Tq, "Tk": w.Tk, "D": w.D,
                   "window": w.window, "recipe": w.recipe, "l2": "256 MB written between calls",
                   "parallelism": f"replicas x{world} (no collective on the data path)"},
        "roofline": {"kernel": "attn_decode (split" + (" + combine)" if per_call > 1 else ")"), "bound": "hbm",
                     "achieved": gbs, "peak": hbm,
                     "unit": "GB/s", "frac": gbs / hbm, "traffic": None, "alg_bytes": nbytes},
        "gpu_launches": per_call * args.steps, "clocks": clocks, "kernel_source_hash": kernel_source_hash(),
    }))
    return 0


PROLOGUE_METRIC = "QK-norm + RoPE prologue HBM GB/s (fwd+bwd, bf16)"


def prologue_bytes(w):
    """Algorithmic bytes of one prologue step, per kernel: the forward reads q, k and writes them back
    normalised and rotated (2 row passes); the backward reads q, k and the output gradients and writes the
    input gradients (3 row passes). A row is D bf16 values."""
    row_bytes = w.B * w.T * (w.H + w.Hkv) * w.D * 2
    return 2 * row_bytes, 3 * row_bytes


def run_prologue(args):
    """QK normalisation + rotary embedding, forward and backward kernels: HBM-bound, measured in GB/s of
    algorithmic bytes against the measured copy bandwidth. The d20 inputs (q, k and their gradients, over
    600 MB) exceed L2, which the line states."""
    from workloads import PROLOGUE_WORKLOADS, make_prologue_inputs
    w = PROLOGUE_WORKLOADS[args.workload]
    rank, world, _ = dist_env()
    fwd_b, bwd_b = prologue_bytes(w)
    if args.impl == "reference":
        if rank != 0:
            return 0
        from threadpoolctl import threadpool_limits

        from oracle import attn_ref
        q, k, gq, gk, offs = make_prologue_inputs(w)
        n, t = min(w.B, 2), min(w.T, 256)
        kw = dict(base=w.rope_base, eps=w.eps, pairing=w.pairing, offsets=0 if offs is None else offs[:n].numpy())
        times = []
        with threadpool_limits(limits=len(os.sched_getaffinity(0))):
            for it in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                for x, g in ((q, gq), (k, gk)):
                    attn_ref.qk_norm_rope(x[:n, :t], **kw)
                    attn_ref.qk_norm_rope_backward(x[:n, :t], g[:n, :t], **kw)
                if it >= args.warmup:
                    times.append(time.perf_counter() - t0)
        frac = (n * t) / (w.B * w.T)
        value = (fwd_b + bwd_b) * frac / (sum(times) / len(times)) / 1e9
        print(json.dumps({"metric": PROLOGUE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
                          "dtype": "f64", "data": "synthetic", "config": {"workload": w.name, "recipe": w.recipe},
                          "cpu_baseline": {"value": value, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
                                           "kind": "oracle",
                                           "sample": f"{n} sequences x {t} positions of {w.name} per step"},
                          "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    import torch

    import causal_self_attention_bf16_b200 as attn
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    q, k, gq, gk, offs = make_prologue_inputs(w, device)
    qo, ko, dq, dk = (torch.empty_like(t) for t in (q, k, q, k))
    lib = attn.load_library()
    sh = torch.cuda.current_stream(device).cuda_stream
    pairing = attn.ROPE_PAIRINGS[w.pairing]
    optr = None if offs is None else offs.data_ptr()

    def fwd():
        st = lib.attn_qk_norm_rope(q.data_ptr(), k.data_ptr(), qo.data_ptr(), ko.data_ptr(), optr, w.B, w.T, w.H,
                                   w.Hkv, w.D, w.rope_base, w.eps, pairing, sh)
        if st != 0:
            raise RuntimeError(f"attn_qk_norm_rope: {attn._STATUS.get(st, st)}")

    def bwd():
        st = lib.attn_qk_norm_rope_bwd(q.data_ptr(), k.data_ptr(), gq.data_ptr(), gk.data_ptr(), dq.data_ptr(),
                                       dk.data_ptr(), optr, w.B, w.T, w.H, w.Hkv, w.D, w.rope_base, w.eps, pairing, sh)
        if st != 0:
            raise RuntimeError(f"attn_qk_norm_rope_bwd: {attn._STATUS.get(st, st)}")

    for _ in range(max(args.warmup, 3)):
        fwd()
        bwd()
    torch.cuda.synchronize(device)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(mk(), mk(), mk()) for _ in range(args.steps)]
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(gpu_id)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    time.sleep(0.1)
    for e0, e1, e2 in ev:
        e0.record()
        fwd()
        e1.record()
        bwd()
        e2.record()
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_f = sum(a.elapsed_time(b) for a, b, _ in ev) / len(ev)
    ms_b = sum(b.elapsed_time(c) for _, b, c in ev) / len(ev)
    ms = reduce_max(ms_f + ms_b, world, device)
    gbs = (fwd_b + bwd_b) / (ms / 1e3) / 1e9
    bwd_gbs = bwd_b / (ms_b / 1e3) / 1e9
    hbm = float(load_peaks()["hbm_gbs"])
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    print(json.dumps({
        "metric": PROLOGUE_METRIC, "value": gbs * world, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "ms_fwd": ms_f, "ms_bwd": ms_b, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "H_kv": w.Hkv, "D": w.D,
                   "pairing": w.pairing, "recipe": w.recipe, "l2": "inputs larger than L2, no flush",
                   "parallelism": f"replicas x{world} (no collective on the data path)"},
        "roofline": {"kernel": "qk_norm_rope_bwd_kernel", "bound": "hbm", "achieved": bwd_gbs, "peak": hbm,
                     "unit": "GB/s", "frac": bwd_gbs / hbm, "alg_bytes": bwd_b,
                     "traffic": recorded_traffic("qk_norm_rope_bwd_kernel", w.name, PROLOGUE_SOURCES)},
        "fwd_roofline": {"kernel": "qk_norm_rope_kernel", "achieved": fwd_b / (ms_f / 1e3) / 1e9,
                         "frac": fwd_b / (ms_f / 1e3) / 1e9 / hbm, "alg_bytes": fwd_b,
                         "traffic": recorded_traffic("qk_norm_rope_kernel", w.name, PROLOGUE_SOURCES)},
        "gpu_launches": 2 * args.steps, "clocks": clocks,
        "kernel_source_hash": kernel_source_hash(PROLOGUE_SOURCES),
    }))
    return 0


def main(argv=None):
    args = parse_args(argv)
    from workloads import DECODE_WORKLOADS, PROLOGUE_WORKLOADS
    if args.workload in DECODE_WORKLOADS:
        return run_decode(args)
    if args.workload in PROLOGUE_WORKLOADS:
        return run_prologue(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
