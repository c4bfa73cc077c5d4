#!/usr/bin/env python
"""Benchmark of tiled GQA prefill attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one launch over the whole workload (every query row of every head):
tfa_prefill (tfa_decode when L <= 8; tfa_attention_ex with a softcap or
sinks; tfa_prefill_ring for a rotating cache; tfa_prefill_varlen for a packed
variable-length batch).  Inputs are seeded synthetic bf16 tensors resident in HBM before
the timed region; L2 is flushed (256 MiB memset) between steps, outside each
step's CUDA events.  Prints one JSON line on rank 0.

Metric: TFLOP/s over allowed (unmasked) pairs, 4*D flops per pair per head.
With --gpus N > 1 (launched by torch.distributed.run) the (batch, KV group)
units of one call are shared by the ranks (sliding_window_gqa_tfa_b200.dist):
--shard weak (default) makes the call N times the workload's batch, so each
rank's share is one copy of the workload on its own inputs; --shard strong
shares the workload's own units.  No data-path collective; the reported time
is the max over ranks.  At N = 1 the line also carries `per_config`: each of
the reference configurations timed the same way, with its max-abs / max-rel
error against the fp64 oracle on the sampled rows the full-size parity test
checks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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
from sliding_window_gqa_tfa_b200.dist import (Run, barrier, max_over_ranks,  # noqa: E402
                                              rank_runs, run_slices, setup, teardown)
from sliding_window_gqa_tfa_b200.flops import workload_bytes, workload_flops  # noqa: E402
from sliding_window_gqa_tfa_b200.inputs import (HEADLINE, WORKLOADS, make_dout,  # noqa: E402
                                                make_inputs, make_sinks, sample_rows, varlen_cu)

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


_NVML_POLLER = """
import signal, sys, time, pynvml
stop = []
signal.signal(signal.SIGTERM, lambda *a: stop.append(1))
pynvml.nvmlInit()
key = sys.argv[1]
h = (pynvml.nvmlDeviceGetHandleByUUID(key) if key.startswith("GPU-")
     else pynvml.nvmlDeviceGetHandleByIndex(int(key)))
get = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
       or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
out = []
t_end = time.time() + 600
while not stop and time.time() < t_end:
    t = time.time()
    try:
        out.append("%.6f %d %d" % (t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), int(get(h))))
    except Exception:
        pass  # a failed query costs one sample, not the record
    time.sleep(0.0002)
print(chr(10).join(out), flush=True)
"""


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: NVML
    polled every ~0.2 ms by a child process (so even a region of a few
    milliseconds gets samples, whatever the launching thread does), each
    sample time-stamped so that only those inside the region [t0, t1] the
    caller marks are summarised; else nvidia-smi at its fastest interval.
    Read-only."""

    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.source = None
        self.samples = []  # (wall time or None, sm MHz, reason bits)
        self.smax = None
        self.region = None  # (t0, t1) of the timed region, wall clock

    def _device_key(self):
        try:  # the same GPU as torch's device, whatever CUDA_VISIBLE_DEVICES says
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            return str(self.idx)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLLER, self._device_key()],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self.proc.stdout.readline().split()  # "max <MHz>": the poller is running
            if len(first) == 2 and first[0] == "max":
                self.smax = float(first[1])
                self.source = "nvml"
                return self
            self.proc.kill()
            self.proc.communicate()
        except OSError:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            return
        time.sleep(0.002)  # a last sample after the region
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in (out or "").splitlines():
            try:
                if self.source == "nvml":
                    t, mhz, bits = line.split()
                    self.samples.append((float(t), float(mhz), int(bits)))
                else:
                    parts = [p.strip() for p in line.split(",")]
                    self.samples.append((None, float(parts[0]), int(parts[2], 16)))
                    self.smax = float(parts[1])
            except (ValueError, IndexError):
                continue

    def summary(self):
        inside = self.samples
        bracketing = False
        if self.region is not None and self.source == "nvml":
            t0, t1 = self.region
            inside = [s_ for s_ in self.samples if t0 <= s_[0] <= t1]
            if not inside:  # one slow NVML query can span a region of a few ms:
                # the samples just before and after it stand in, and the line says so
                before = [s_ for s_ in self.samples if s_[0] < t0]
                after = [s_ for s_ in self.samples if s_[0] > t1]
                inside = before[-1:] + after[:1]
                bracketing = bool(inside)
        pairs = [(mhz, r) for _, mhz, r in inside]
        load = [(mhz, r) for mhz, r in pairs if not (r & 0x1)]  # not GPU-idle
        use = load or pairs
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": self.smax, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = sorted({n for _, r in use for bit, n in self.REASONS.items() if r & bit})
        out = {"sm_mhz": statistics.median(m for m, _ in use), "sm_max_mhz": self.smax,
               "reasons": reasons, "samples": len(pairs), "samples_under_load": len(load),
               "source": self.source}
        if bracketing:
            out["bracketing_samples"] = True  # none fell inside the timed region itself
        return out


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def rows_flops(L, S, causal, window, D, i):
    """Useful flops of query rows i (0 <= i < L) of one head: 4*D per key the row
    may see under causal/window (a key mask is ignored in the count)."""
    P = S - L
    if causal:
        last = np.minimum(P + i, S - 1)
        first = np.maximum(0, last - window + 1) if window > 0 else np.zeros_like(i)
        keys = np.maximum(last - first + 1, 0)
    else:
        keys = np.full_like(i, S)
    return int(keys.sum()) * 4 * D


def workload_config(w):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "S": w.S, "D": w.D,
            "causal": w.causal, "window": w.window, "key_mask": w.key_mask_keep is not None,
            "softcap": w.softcap, "sinks": w.sink_scale is not None, "ring_rows": w.ring_rows,
            "varlen_tokens": sum(L for L, _ in w.seqlens) if w.seqlens else None}


class OracleSampler:
    """Bounded units of the fp64 oracle's work on a workload: a few random query
    rows (of a random sequence, for a packed variable-length workload)."""

    def __init__(self, w, seed=0):
        import oracle

        oracle.build()
        self.oracle, self.w = oracle, w
        self.q, self.k, self.v, self.km = make_inputs(w, seed=seed)
        self.sinks = make_sinks(w, seed=seed)
        if w.kind == "varlen":
            self.cq, self.ck = varlen_cu(w)
            self.live = [b for b, (L, _) in enumerate(w.seqlens) if L > 0]
        self.n_rows = w.B * w.Hq * w.L
        if w.kind == "backward":
            self.dout = make_dout(w, seed=seed)

    def unit(self, rng, n):
        """Run the oracle on n random rows; return their useful flops."""
        w, o = self.w, self.oracle
        kw = dict(scale=w.softmax_scale, window=w.window, softcap=w.softcap, sinks=self.sinks)
        if w.kind == "backward":
            # the gradients of n query rows of one KV group (all heads of the
            # group), over the keys those rows reach: a sub-problem of the same
            # shape family (prefix S - L kept), rows starting at a random tile
            G = w.Hq // w.Hkv
            P = w.S - w.L
            r0 = int(rng.integers(0, max(1, w.L - n + 1)))
            rows = slice(r0, r0 + n)
            g = int(rng.integers(0, w.Hkv))
            heads = slice(g * G, (g + 1) * G)
            S_sub = P + r0 + n
            q = self.q[:1, heads, rows].contiguous()
            do = self.dout[:1, heads, rows].contiguous()
            k = self.k[:1, g:g + 1, :S_sub].contiguous()
            v = self.v[:1, g:g + 1, :S_sub].contiguous()
            # rows r0..r0+n-1 of the full problem are rows 0..n-1 here with prefix P + r0
            o.attention_backward(q, k, v, do, scale=w.softmax_scale, causal=w.causal, window=w.window)
            return 10 * w.D * G * int(sum(min(P + r0 + i, S_sub - 1) + 1 -
                                          (max(0, P + r0 + i - w.window + 1) if w.window > 0 else 0)
                                          for i in range(n)) if w.causal else n * S_sub * G * 10 * w.D)
        if w.kind == "varlen":
            # one sequence through the dense oracle (the varlen definition per sequence)
            b = int(rng.choice(self.live))
            L, S = w.seqlens[b]
            qb = self.q[self.cq[b]:self.cq[b + 1]].transpose(0, 1)[None].contiguous()
            kb = self.k[self.ck[b]:self.ck[b + 1]].transpose(0, 1)[None].contiguous()
            vb = self.v[self.ck[b]:self.ck[b + 1]].transpose(0, 1)[None].contiguous()
            rows = np.sort(rng.choice(w.Hq * L, size=min(n, w.Hq * L), replace=False)).astype(np.int64)
            o.attention(qb, kb, vb, causal=w.causal, rows=rows, **kw)
            return rows_flops(L, S, w.causal, w.window, w.D, rows % L)
        rows = np.sort(rng.choice(self.n_rows, size=min(n, self.n_rows), replace=False)).astype(np.int64)
        if w.kind == "ring":
            o.attention_ring(self.q, self.k, self.v, S=w.S, rows=rows, **kw)
        else:
            o.attention(self.q, self.k, self.v, causal=w.causal, key_mask=self.km, rows=rows, **kw)
        return rows_flops(w.L, w.S, w.causal, w.window, w.D, rows % w.L)


def cpu_baseline(w, budget_s=12.0):
    """The fp64 oracle as it stands, on the host cores, over a bounded row sample."""
    sampler = OracleSampler(w, seed=0)
    rng = np.random.default_rng(0)
    chunk = 64
    done_rows, flops, t0 = 0, 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        flops += sampler.unit(rng, chunk)
        done_rows += chunk
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{done_rows} random query rows of {w.name} (of {sampler.n_rows}), fp64, "
                      f"{dt:.1f} s wall; flops counted as 4*D per key the row may see "
                      f"(key mask ignored in the count)"}


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sampler = OracleSampler(w, seed=0)
    rng = np.random.default_rng(1)
    per_step = 8 if w.kind == "backward" else 32  # the backward oracle runs one KV group per thread
    times, flops = [], []
    for step in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        f = sampler.unit(rng, per_step)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
            flops.append(f)
    total_t = sum(times)
    value = sum(flops) / total_t / 1e12
    sample = (f"each step: {per_step} random query rows of {w.name} through the fp64 oracle "
              f"on {cpu_threads()} host threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**workload_config(w), "sample_rows_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# The reference configurations timed beside the headline at N = 1 (the workload
# the metric is quoted on is the headline line itself; its error is reported too).
PER_CONFIG = ["witness_33x47", "qwen3_prefill_b4_2048", HEADLINE, "llama_gqa_chunk_2048x8192_keymask",
              "swa_rotating_w1024_2048", "long_chunk_2048x32768", "long_chunk_2048x32768_d64",
              "bidirectional_4096"]


def oracle_errors(w, o, q, k, v, km):
    """Max-abs / max-rel error of the bf16 output o (on the device) against the
    fp64 oracle on the rows the full-size parity test samples (every row of a
    tiny workload), and the worst ratio of the error to the tolerance
    0.02 + 0.02 |ref| (<= 1 passes).  Relative error over |ref| >= 0.05."""
    import oracle

    oracle.build()
    tiny = w.B * w.Hq * w.L <= 4096
    rows = None if tiny else sample_rows(w, n_per_head=12 if w.S >= 16384 else 24)
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km, softcap=w.softcap, sinks=make_sinks(w, 0), rows=rows)
    got = o.reshape(-1, w.D) if rows is not None else o
    if rows is not None:
        got = got[torch.as_tensor(rows, device=o.device)]
    got = got.float().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(got - ref)
    big = np.abs(ref) >= 0.05
    return {"max_abs_err": float(err.max()),
            "max_rel_err": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
            "worst_tol_ratio": float((err / (0.02 + 0.02 * np.abs(ref))).max()),
            "rows_checked": int(ref.reshape(-1, w.D).shape[0])}


def time_launches(step, flush, stream, steps, warmup, dev, world=1):
    """Per-launch device times (ms) of `steps` launches after `warmup`, L2 flushed
    before each, CUDA events on the launching stream; clocks sampled meanwhile.
    The sampler starts before the warm-up, so that the GPU does not sit idle
    while it starts between the warm-up and the timed launches (after such a
    gap the first timed launches ran slower on some boxes); only samples inside
    the timed region are kept."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(warmup):
            flush.zero_()
            step()
        tb.check_status(stream)
        barrier(world)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter()
        r0 = time.time()
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        clk.region = (r0, time.time())
        t_wall = time.perf_counter() - t_wall
    barrier(world)
    tb.check_status(stream)
    return [s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)], clk.summary(), t_wall


def per_config(args, dev, flush, stream, peaks):
    """Each reference configuration: device time (as the headline), throughput,
    fraction of the measured peak, clocks, and error against the fp64 oracle."""
    res = {}
    for name in PER_CONFIG:
        w = WORKLOADS[name]
        q, k, v, km = make_inputs(w, seed=0)
        dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
        dkm = km.to(dev) if km is not None else None
        o = torch.empty_like(dq)

        def step():
            tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=w.causal, window=w.window,
                       key_mask=dkm, out=o)

        per, clocks, _ = time_launches(step, flush, stream, args.steps, args.warmup, dev)
        per = sorted(per)
        mean = sum(per) / len(per)
        fl = workload_flops(w, key_mask=km)
        tflops = fl / (mean * 1e-3) / 1e12
        res[name] = {"ms_mean": mean, "ms_p50": per[len(per) // 2], "tflops": tflops,
                     "frac": tflops / float(peaks["bf16_tflops"]), "useful_gflop": fl / 1e9,
                     "clock_sm_mhz": clocks["sm_mhz"], "clock_reasons": clocks["reasons"],
                     **oracle_errors(w, o, q, k, v, km)}
        del dq, dk, dv, dkm, o
        torch.cuda.empty_cache()
    return res


def bench_runs(w, world, rank, strong):
    """The runs (dist.Run, element indices local to this rank's tensors) a rank
    launches per step.  Strong: its share of the workload's own B x Hkv units
    (every rank holds the whole call's inputs).  Weak: a call of world x B
    elements whose share for this rank is exactly its own B elements (its own
    inputs), so the runs are shifted to local element indices."""
    if strong:
        return rank_runs(w.B, w.Hkv, world, rank)
    return [Run(r_.b0 - rank * w.B, r_.nb, r_.g0, r_.ng) for r_ in rank_runs(world * w.B, w.Hkv, world, rank)]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="tfa", choices=["tfa", "reference"])
    ap.add_argument("--shard", default="weak", choices=["weak", "strong"],
                    help="N > 1: one call N times the workload's batch (weak) or the workload "
                         "itself (strong), its (batch, KV group) units shared by the ranks")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    world, rank, local = setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    tb.lib()  # fail loudly if the library is missing

    # Dense workloads at N > 1 run this rank's share of one call's (batch, KV
    # group) units; the other kinds run one copy of the workload per rank.
    strong = world > 1 and args.shard == "strong" and w.kind == "dense"
    seed = 0 if strong else rank  # a strong-scaling call's inputs are the same on every rank
    q, k, v, km = make_inputs(w, seed=seed)
    sinks = make_sinks(w, seed=seed)
    if w.kind == "varlen":
        extra = tuple(torch.from_numpy(c) for c in varlen_cu(w))
    elif w.kind == "backward":
        extra = (make_dout(w, seed=rank),)
    else:
        extra = ()
    host_inputs = [q, k, v, km, sinks, *extra]  # what one call reads (None: absent)
    dev_inputs = [t.to(dev) if t is not None else None for t in host_inputs]
    if w.saved_stats:  # the forward's output and log-sum-exp, made once before any timing
        o_saved, lse_saved = tb.prefill_lse(*dev_inputs[:3], scale=w.softmax_scale, causal=w.causal,
                                            window=w.window, key_mask=dev_inputs[3])
        torch.cuda.synchronize(dev)
        host_inputs += [o_saved.cpu(), lse_saved.cpu()]
        dev_inputs += [o_saved, lse_saved]
    if w.kind == "backward":  # (dq, dk, dv)
        out = tuple(torch.empty_like(t) for t in dev_inputs[:3])
    else:
        out = torch.empty_like(dev_inputs[0])
    G = w.Hq // w.Hkv
    if w.kind == "dense":
        runs = bench_runs(w, world, rank, strong)
        flops = sum(workload_flops(w.with_(B=r_.nb, Hq=r_.ng * G, Hkv=r_.ng),
                                   key_mask=km[r_.b0:r_.b0 + r_.nb] if km is not None else None)
                    for r_ in runs)
    else:
        runs = None
        flops = workload_flops(w, key_mask=km)
    call_flops = workload_flops(w, key_mask=km)  # one copy of the workload
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call(ins, o):
        """One step on the current stream: the entry point the workload needs
        (for a dense workload, one call per run of this rank's units)."""
        dq, dk, dv, dkm, dsinks = ins[:5]
        if w.kind == "backward":
            tb.backward(dq, dk, dv, ins[5], scale=w.softmax_scale, causal=w.causal, window=w.window,
                        key_mask=dkm, out=o, saved=(ins[6], ins[7]) if w.saved_stats else None)
        elif w.kind == "varlen":
            tb.prefill_varlen(dq, dk, dv, ins[5], ins[6], max_seqlen_q=w.L, scale=w.softmax_scale,
                              causal=w.causal, window=w.window, softcap=w.softcap, sinks=dsinks,
                              out=o)
        elif w.kind == "ring":
            tb.prefill_ring(dq, dk, dv, S=w.S, window=w.window, scale=w.softmax_scale,
                            softcap=w.softcap, sinks=dsinks, out=o)
        else:
            for r_ in runs:
                (qb, qh), (kb, kh) = run_slices(r_, G)
                tb.prefill(dq[qb, qh], dk[kb, kh], dv[kb, kh], scale=w.softmax_scale,
                           causal=w.causal, window=w.window,
                           key_mask=dkm[qb] if dkm is not None else None, out=o[qb, qh],
                           softcap=w.softcap, sinks=dsinks[qh] if dsinks is not None else None)

    def step():
        call(dev_inputs, out)

    per, clocks, t_wall = time_launches(step, flush, stream, args.steps, args.warmup, dev, world)
    mean_ms = sum(per) / len(per)
    mean_ms = max_over_ranks(mean_ms, world)
    # whole-job throughput: every rank's units over the slowest rank's time
    job_flops = call_flops if strong else flops * world
    value = job_flops / (mean_ms * 1e-3) / 1e12
    per_sorted = sorted(per)

    # L2-warm reference (no flush between launches; the inputs of the previous
    # launch may still be in L2): reported beside the flushed headline, not in it
    n_warm = min(args.steps, 50)
    w_starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_warm)]
    w_ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_warm)]
    for i in range(n_warm):
        w_starts[i].record(stream)
        step()
        w_ends[i].record(stream)
    torch.cuda.synchronize(dev)
    tb.check_status(stream)
    warm_sorted = sorted(s_.elapsed_time(e_) for s_, e_ in zip(w_starts, w_ends))
    warm_ms = max_over_ranks(warm_sorted[len(warm_sorted) // 2], world)
    errors = oracle_errors(w, out, q, k, v, km) if (w.kind == "dense" and world == 1) else None

    # end to end through the C ABI with host buffers (copies inside the timed region)
    pinned = [t.pin_memory() if t is not None else None for t in host_inputs]
    hq, hk, hv, hkm = pinned[:4]
    if w.kind == "backward":
        hout = tuple(torch.empty_like(t).pin_memory() for t in (hq, hk, hv))
    else:
        hout = torch.empty_like(hq).pin_memory()
    if w.kind != "dense" or w.softcap > 0 or sinks is not None:
        # the device entry points: the step copies the pinned inputs in, calls
        # the entry point, and copies the output back, all on `stream`
        staged = [torch.empty_like(t) if t is not None else None for t in dev_inputs]
        eout = tuple(torch.empty_like(t) for t in out) if w.kind == "backward" else torch.empty_like(out)

        def e2e_step():
            for d, h in zip(staged, pinned):
                if d is not None:
                    d.copy_(h, non_blocking=True)
            call(staged, eout)
            for h, d in (zip(hout, eout) if w.kind == "backward" else [(hout, eout)]):
                h.copy_(d, non_blocking=True)
        entry = {"varlen": "tfa_prefill_varlen", "ring": "tfa_prefill_ring",
                 "backward": "tfa_prefill_backward_saved" if w.saved_stats else "tfa_prefill_backward"
                 }.get(w.kind, "tfa_attention_ex")
        e2e_api = f"{entry} (pinned host buffers, copies on the stream)"
        h2d = sum(t.numel() * t.element_size() for t in pinned if t is not None)
    else:
        def e2e_step():
            for r_ in runs:  # this rank's share, from and to host buffers
                (qb, qh), (kb, kh) = run_slices(r_, G)
                tb.prefill_host(hq[qb, qh], hk[kb, kh], hv[kb, kh], scale=w.softmax_scale,
                                causal=w.causal, window=w.window,
                                key_mask=hkm[qb] if hkm is not None else None, out=hout[qb, qh],
                                stream=stream)
        e2e_api = "tfa_prefill_host (pinned host buffers)"
        h2d = sum(hq[run_slices(r_, G)[0]].numel() * 2 + 2 * hk[run_slices(r_, G)[1]].numel() * 2 +
                  (hkm[r_.b0:r_.b0 + r_.nb].numel() * 4 if hkm is not None else 0) for r_ in runs)
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
    if runs is not None:
        d2h = sum(hout[run_slices(r_, G)[0]].numel() * 2 for r_ in runs)
    else:
        d2h = sum(t.numel() * 2 for t in hout) if w.kind == "backward" else hout.numel() * 2

    peaks, peak_kind = load_peaks()
    alg_bytes = workload_bytes(w)
    if w.L <= tb.MAX_DECODE_ROWS:
        # short queries read every K/V byte for a few flops: bounded by HBM
        bound, roof_unit = "hbm", "GB/s"
        peak = float(peaks["hbm_gbs"])
        achieved = alg_bytes * flops / call_flops / (mean_ms * 1e-3) / 1e9
        peak_source = f"{peak_kind} hbm_gbs (copy bandwidth)"
    else:
        bound, roof_unit = "tensor", "TFLOP/s"
        peak = float(peaks["bf16_tflops"])
        achieved = flops / (mean_ms * 1e-3) / 1e12  # per GPU, per launch
        peak_source = f"{peak_kind} bf16_tflops (burst; kernel timed alone)"
    traffic = recorded_traffic(w.name) if (world == 1 or not strong) else None
    n_calls = len(runs) if runs is not None else 1
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
            "higher_is_better": True, "scaling": "strong" if strong else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(w), "useful_gflop": job_flops / 1e9,
                       "l2": "flushed between steps (256 MiB memset outside the step events)",
                       "parallelism": ("single GPU" if world == 1 else
                                       f"(batch, KV group) units of one call over {world} GPUs: "
                                       + ("the workload's own call (strong)" if strong else
                                          f"a call of {world} x B elements, one copy per GPU (weak)"))},
            "ms_p10": per_sorted[len(per) // 10], "ms_p50": per_sorted[len(per) // 2],
            "ms_p90": per_sorted[(9 * len(per)) // 10],
            "l2_warm": {"ms_p50": warm_ms, "value": job_flops / (warm_ms * 1e-3) / 1e12,
                        "unit": UNIT, "launches": n_warm},
            "pct_of_peak": 100.0 * achieved / peak,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                         "unit": roof_unit, "frac": achieved / peak,
                         "peak_source": peak_source,
                         "traffic": traffic,
                         "algorithmic_bytes": alg_bytes},
            "e2e": {"value": job_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "api": e2e_api},
            # kernels per step: one per call, or four for the backward (forward
            # recompute, delta, dQ, dK/dV), three when it starts from the saved statistics
            "gpu_launches": args.steps * ((3 if w.saved_stats else 4) if w.kind == "backward" else n_calls),
            "clocks": clocks,
            "wall_s_timed_region": t_wall,
        }
        if errors is not None:
            line["error_vs_oracle"] = errors
        if world == 1 and not args.no_per_config and w.name == HEADLINE:
            line["per_config"] = per_config(args, dev, flush, stream, peaks)
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    teardown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
