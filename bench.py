#!/usr/bin/env python
"""Benchmark of tiled GQA prefill attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one launch (tfa_prefill; tfa_decode when L <= 8) over the whole workload (every query row of
every head).  Inputs are seeded synthetic bf16 tensors resident in HBM before
the timed region; L2 is flushed (256 MiB memset) between steps, outside each
step's CUDA events.  Prints one JSON line on rank 0.

Metric: TFLOP/s over allowed (unmasked) pairs, 4*D flops per pair per head.
With --gpus N > 1 (launched by torch.distributed.run) every rank runs the same
workload on its own inputs (weak scaling, no data-path collective); the
reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sliding_window_gqa_tfa_b200 import binding as tb  # noqa: E402
from sliding_window_gqa_tfa_b200.flops import algorithmic_bytes, useful_flops  # noqa: E402
from sliding_window_gqa_tfa_b200.inputs import HEADLINE, WORKLOADS, make_inputs, make_sinks  # noqa: E402

METRIC = "prefill attention TFLOP/s (unmasked pairs) and % of B200 BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_NAME = "tfa_prefill_kernel"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sliding_window_gqa_tfa_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{KERNEL_NAME}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return int(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rows_flops(w, rows):
    """Useful flops of the given flattened rows (host arithmetic, 4*D per allowed key)."""
    i = rows % w.L
    P = w.S - w.L
    if w.causal:
        last = P + i
        first = np.maximum(0, last - w.window + 1) if w.window > 0 else np.zeros_like(i)
        keys = last - first + 1
    else:
        keys = np.full_like(i, w.S)
    return int(keys.sum()) * 4 * w.D


def cpu_baseline(w, q, k, v, km, budget_s=12.0):
    """The fp64 oracle as it stands, on the host cores, over a bounded row sample."""
    import oracle

    oracle.build()
    rng = np.random.default_rng(0)
    n_rows = w.B * w.Hq * w.L
    chunk = 64
    done_rows, flops, t0 = 0, 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        rows = np.sort(rng.choice(n_rows, size=chunk, replace=False)).astype(np.int64)
        oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                         key_mask=km, softcap=w.softcap, sinks=make_sinks(w, 0), rows=rows)
        done_rows += chunk
        flops += oracle_rows_flops(w, rows)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{done_rows} random query rows of {w.name} (of {n_rows}), fp64, "
                      f"{dt:.1f} s wall; flops counted as 4*D per key the row may see "
                      f"(key mask ignored in the count)"}


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    q, k, v, km = make_inputs(w, seed=0)
    sinks = make_sinks(w, seed=0)
    rng = np.random.default_rng(1)
    n_rows = w.B * w.Hq * w.L
    per_step = 32
    times, flops = [], []
    for step in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(n_rows, size=per_step, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                         key_mask=km, softcap=w.softcap, sinks=sinks, rows=rows)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
            flops.append(oracle_rows_flops(w, rows))
    total_t = sum(times)
    value = sum(flops) / total_t / 1e12
    sample = (f"each step: {per_step} random query rows of {w.name} through the fp64 oracle "
              f"on {cpu_threads()} host threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L,
                       "S": w.S, "D": w.D, "causal": w.causal, "window": w.window,
                       "key_mask": w.key_mask_keep is not None, "softcap": w.softcap,
                       "sinks": w.sink_scale is not None, "sample_rows_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="tfa", choices=["tfa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    tb.lib()  # fail loudly if the library is missing

    q, k, v, km = make_inputs(w, seed=rank)
    sinks = make_sinks(w, seed=rank)
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    dkm = km.to(dev) if km is not None else None
    dsinks = sinks.to(dev) if sinks is not None else None
    variant = w.softcap > 0 or sinks is not None  # score variants: tfa_attention_ex
    out = torch.empty_like(dq)
    flops = useful_flops(w.B, w.Hq, w.L, w.S, w.D, causal=w.causal, window=w.window, key_mask=km)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=w.causal, window=w.window,
                   key_mask=dkm, out=out, softcap=w.softcap, sinks=dsinks)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    tb.check_status(stream)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall
    barrier(world)
    tb.check_status(stream)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]  # ms
    mean_ms = sum(per) / len(per)
    mean_ms = max_over_ranks(mean_ms, world)
    value = flops * world / (mean_ms * 1e-3) / 1e12
    per_sorted = sorted(per)

    # end to end through the C ABI with host buffers (copies inside the timed region)
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hkm = km.pin_memory() if km is not None else None
    hout = torch.empty_like(hq).pin_memory()
    hsinks = sinks.pin_memory() if sinks is not None else None
    if variant:
        # tfa_attention_ex takes device pointers: the step copies the pinned
        # inputs in, calls it, and copies the output back, all on `stream`
        eq, ek, ev = torch.empty_like(dq), torch.empty_like(dk), torch.empty_like(dv)
        ekm = torch.empty_like(dkm) if dkm is not None else None
        esinks = torch.empty_like(dsinks) if dsinks is not None else None
        eout = torch.empty_like(dq)

        def e2e_step():
            for d, h in ((eq, hq), (ek, hk), (ev, hv), (ekm, hkm), (esinks, hsinks)):
                if d is not None:
                    d.copy_(h, non_blocking=True)
            tb.prefill(eq, ek, ev, scale=w.softmax_scale, causal=w.causal, window=w.window,
                       key_mask=ekm, out=eout, softcap=w.softcap, sinks=esinks)
            hout.copy_(eout, non_blocking=True)
        e2e_api = "tfa_attention_ex (pinned host buffers, copies on the stream)"
    else:
        def e2e_step():
            tb.prefill_host(hq, hk, hv, scale=w.softmax_scale, causal=w.causal, window=w.window,
                            key_mask=hkm, out=hout, stream=stream)
        e2e_api = "tfa_prefill_host (pinned host buffers)"
    for _ in range(3):
        e2e_step()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2 + (hkm.numel() * 4 if hkm is not None else 0) \
        + (hsinks.numel() * 4 if hsinks is not None else 0)
    d2h = hout.numel() * 2

    peaks, peak_kind = load_peaks()
    alg_bytes = algorithmic_bytes(w.B, w.Hq, w.Hkv, w.L, w.S, w.D, key_mask=km is not None)
    if w.L <= tb.MAX_DECODE_ROWS:
        # short queries read every K/V byte for a few flops: bounded by HBM
        bound, roof_unit = "hbm", "GB/s"
        peak = float(peaks["hbm_gbs"])
        achieved = alg_bytes / (mean_ms * 1e-3) / 1e9
        peak_source = f"{peak_kind} hbm_gbs (copy bandwidth)"
    else:
        bound, roof_unit = "tensor", "TFLOP/s"
        peak = float(peaks["bf16_tflops"])
        achieved = flops / (mean_ms * 1e-3) / 1e12  # per GPU, per launch
        peak_source = f"{peak_kind} bf16_tflops (burst; kernel timed alone)"
    traffic = recorded_traffic(w.name)
    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L,
                       "S": w.S, "D": w.D, "causal": w.causal, "window": w.window,
                       "key_mask": w.key_mask_keep is not None, "softcap": w.softcap,
                       "sinks": w.sink_scale is not None, "useful_gflop": flops / 1e9,
                       "l2": "flushed between steps (256 MiB memset outside the step events)",
                       "parallelism": f"weak x{world}" if world > 1 else "single GPU"},
            "ms_p10": per_sorted[len(per) // 10], "ms_p50": per_sorted[len(per) // 2],
            "ms_p90": per_sorted[(9 * len(per)) // 10],
            "pct_of_peak": 100.0 * achieved / peak,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                         "unit": roof_unit, "frac": achieved / peak,
                         "peak_source": peak_source,
                         "traffic": traffic,
                         "algorithmic_bytes": alg_bytes},
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "api": e2e_api},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "wall_s_timed_region": t_wall,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w, q, k, v, km)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
