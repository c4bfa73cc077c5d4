"""Host arithmetic behind the bench line, checked on the CPU.

The throughput metric counts 4*D flops per allowed (b, h, row, key) pair: here
the closed form per key (flops.allowed_pairs) and the per-row form the CPU
baseline uses (bench.rows_flops) are compared with a brute-force count of the
definition (causal: key j <= S-L+i; window: j > S-L+i-W; key mask kept), and
the algorithmic bytes with the sizes of the tensors the input generator
actually makes.  The clock record's summary (timed-region filter, idle
samples, throttle-reason bits, the bracketing fallback) and the profile gate
of `roofline.traffic` run on synthetic data.
"""
import numpy as np
import pytest

import bench
from sliding_window_gqa_tfa_b200.flops import allowed_pairs, workload_bytes, workload_flops
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped


def _brute_pairs(B, Hq, L, S, causal, window, km):
    P = S - L
    i = np.arange(L)[:, None]
    j = np.arange(S)[None, :]
    vis = np.ones((L, S), dtype=bool)
    if causal:
        vis &= j <= P + i
        if window > 0:
            vis &= j > P + i - window
    total = 0
    for b in range(B):
        keep = np.ones(S, dtype=bool) if km is None else km[b] > 0.5
        total += int((vis & keep[None, :]).sum())
    return total * Hq


@pytest.mark.parametrize("B,Hq,L,S,causal,window,keep", [
    (1, 2, 33, 47, True, 0, None),
    (2, 3, 130, 700, True, 129, None),
    (1, 4, 300, 300, True, 1, None),        # window 1: the diagonal only
    (2, 2, 50, 400, False, 0, None),
    (3, 1, 200, 450, True, 100, 0.6),
    (1, 2, 8, 9000, True, 0, 0.1),
])
def test_allowed_pairs_match_the_definition(B, Hq, L, S, causal, window, keep):
    km = None
    if keep is not None:
        km = (np.random.default_rng(1).random((B, S)) < keep).astype(np.float32)
    want = _brute_pairs(B, Hq, L, S, causal, window, km)
    assert allowed_pairs(B, Hq, L, S, causal=causal, window=window, key_mask=km) == want


@pytest.mark.parametrize("L,S,causal,window", [(33, 47, True, 0), (300, 1000, True, 257),
                                                (64, 64, False, 0), (129, 129, True, 0)])
def test_row_flops_sum_to_the_head_total(L, S, causal, window):
    rows = np.arange(L)
    assert bench.rows_flops(L, S, causal, window, 128, rows) == \
        4 * 128 * _brute_pairs(1, 1, L, S, causal, window, None)
    # and split into two disjoint row sets
    a, b = rows[rows % 3 == 0], rows[rows % 3 != 0]
    assert bench.rows_flops(L, S, causal, window, 64, a) + bench.rows_flops(L, S, causal, window, 64, b) \
        == bench.rows_flops(L, S, causal, window, 64, rows)


def test_varlen_and_backward_flops():
    w = WORKLOADS["varlen_qwen3_16seqs"]
    want = sum(4 * w.D * _brute_pairs(1, w.Hq, L, S, w.causal, w.window or 0, None)
               for L, S in w.seqlens[:3])
    part = w.with_(seqlens=w.seqlens[:3])
    assert workload_flops(part) == want
    fwd = WORKLOADS["llama_gqa_chunk_2048x8192"]
    bwd = WORKLOADS["llama_gqa_chunk_2048x8192_backward"]
    assert 2 * workload_flops(bwd) == 5 * workload_flops(fwd)  # five products of 2*D against two


@pytest.mark.parametrize("w", [shaped(2, 6, 3, 40, 90, 64), shaped(1, 8, 2, 33, 47, 128, key_mask_keep=0.5)],
                         ids=["plain", "key_mask"])
def test_algorithmic_bytes_are_the_tensors_touched_once(w):
    q, k, v, km = make_inputs(w, seed=3)
    nbytes = lambda t: t.numel() * t.element_size()
    want = 2 * nbytes(q) + nbytes(k) + nbytes(v) + (nbytes(km) if km is not None else 0)  # O like Q
    assert workload_bytes(w) == want


def _sampler(samples, region, smax=1965.0):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.idx, s.proc, s.source, s.smax = 0, None, "nvml", smax
    s.samples, s.region = samples, region
    return s


def test_clock_summary_keeps_the_timed_region_and_load():
    samples = [(0.5, 1200.0, 0x1),            # before the region, idle
               (1.1, 1965.0, 0x0), (1.2, 1950.0, 0x4), (1.3, 1965.0, 0x1),
               (2.5, 900.0, 0x40)]            # after the region: ignored
    out = _sampler(samples, (1.0, 2.0)).summary()
    assert out["samples"] == 3 and out["samples_under_load"] == 2
    assert out["sm_mhz"] == pytest.approx((1965.0 + 1950.0) / 2)
    assert out["reasons"] == ["sw_power_cap"]
    assert "bracketing_samples" not in out


def test_clock_summary_decodes_every_reason_bit():
    bits = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    for bit, name in bits.items():
        out = _sampler([(1.5, 1800.0, bit)], (1.0, 2.0)).summary()
        assert out["reasons"] == [name]


def test_clock_summary_brackets_a_region_without_samples():
    samples = [(0.9, 1965.0, 0x0), (0.95, 1960.0, 0x0), (2.1, 1950.0, 0x0), (2.2, 1000.0, 0x0)]
    out = _sampler(samples, (1.0, 2.0)).summary()
    assert out["bracketing_samples"] is True
    assert out["samples"] == 2 and out["sm_mhz"] == pytest.approx((1960.0 + 1950.0) / 2)
    empty = _sampler([], (1.0, 2.0)).summary()
    assert empty["samples"] == 0 and empty["sm_mhz"] is None


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / f"{bench.KERNEL_NAME}_some_workload.md").write_text(
        "# summary\n\nkernel_source_sha: 0123456789abcdef\ndram_bytes_per_launch: 4242\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0123456789abcdef")
    assert bench.recorded_traffic("some_workload") == 4242
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "fedcba9876543210")
    assert bench.recorded_traffic("some_workload") is None   # the kernel changed since
    assert bench.recorded_traffic("other_workload") is None  # no capture at all


def test_kernel_source_hash_follows_the_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "sliding_window_gqa_tfa_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_source_hash()
    (csrc / "a.cu").write_text("y")
    h2 = bench.kernel_source_hash()
    assert len(h1) == 16 and h1 != h2
