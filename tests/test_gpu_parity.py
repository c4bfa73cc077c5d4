"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on
the same seeded inputs.

Bar: |gpu - oracle| <= 0.02 + 0.02 |oracle| element-wise on the bf16 output
(the operator tolerance of tiny-llm "Week 2 Day 5: Tiled Dense Prefill
Attention", Task 1: atol = rtol = 0.02).  Small cases compare every element;
the full-size workloads, launched exactly as the benchmark launches them,
compare sampled rows that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, make_sinks, sample_rows, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    tb.lib()  # raises if the library is missing: no fallback


def _run(w, seed=0, flags=0, inputs=None):
    q, k, v, km = inputs if inputs is not None else make_inputs(w, seed)
    sinks = make_sinks(w, seed)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dkm = km.cuda() if km is not None else None
    o = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=w.causal, window=w.window,
                   key_mask=dkm, debug_flags=flags, softcap=w.softcap,
                   sinks=sinks.cuda() if sinks is not None else None)
    tb.check_status()
    return o, (q, k, v, km)


def _assert_close(got, ref, what):
    got = got.float().cpu().double().numpy() if isinstance(got, torch.Tensor) else got
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, "
                           f"max abs err {err.max():.4g}")
    return float(err.max())


SMALL = [
    ("witness_33x47", WORKLOADS["witness_33x47"]),
    ("min_rows_9x9", shaped(1, 4, 2, 9, 9, 128)),
    ("ragged_130x300", shaped(2, 4, 2, 130, 300, 128)),
    ("pair_tail_257x257", shaped(1, 2, 1, 257, 257, 128)),
    ("exact_256x512", shaped(1, 2, 2, 256, 512, 128)),
    ("three_pairs_600x700", shaped(1, 3, 3, 600, 700, 128)),
    ("group7_200x450", shaped(1, 14, 2, 200, 450, 128)),
    ("window1", shaped(1, 4, 2, 140, 400, 128, window=1)),
    ("window127", shaped(1, 4, 2, 300, 700, 128, window=127)),
    ("window128", shaped(1, 4, 2, 300, 700, 128, window=128)),
    ("window129", shaped(1, 4, 2, 300, 700, 128, window=129)),
    ("window_rotating_small", shaped(1, 4, 2, 256, 1023 + 256, 128, window=1024)),
    ("window_wider_than_S", shaped(1, 4, 2, 100, 200, 128, window=5000)),
    ("bidirectional_ragged", shaped(2, 4, 2, 100, 333, 128, causal=False)),
    ("keymask_causal", shaped(2, 4, 2, 150, 400, 128, key_mask_keep=0.9)),
    ("keymask_sparse", shaped(1, 4, 2, 140, 300, 128, key_mask_keep=0.05)),
    ("keymask_window", shaped(1, 4, 2, 200, 500, 128, window=100, key_mask_keep=0.5)),
    ("keymask_bidir", shaped(1, 4, 4, 64, 200, 128, causal=False, key_mask_keep=0.7)),
    ("sharp_softmax", shaped(1, 4, 2, 200, 600, 128, k_scale=4.0)),
    ("d64_witness", shaped(1, 8, 2, 33, 47, 64)),
    ("d64_ragged", shaped(2, 4, 2, 130, 300, 64)),
    ("d64_window", shaped(1, 4, 2, 300, 700, 64, window=129)),
    ("d64_keymask_bidir", shaped(1, 4, 2, 100, 250, 64, causal=False, key_mask_keep=0.8)),
    # chunks of at most 128 rows run packed: a 128-row tile holds the rows of
    # floor(128 / L) query heads of one KV group (the last tile of a group may
    # hold fewer), and long key ranges are cut over several CTAs whose partials
    # the first piece merges with its whole warpgroup
    ("pack3_of4_L40_long", shaped(1, 8, 2, 40, 3000, 128)),
    ("pack2_L64_window", shaped(2, 8, 2, 64, 2000, 128, window=300)),
    ("pack5_of6_L24_keymask_d64", shaped(1, 12, 2, 24, 900, 64, key_mask_keep=0.7)),
    ("pack8_L16_bidir", shaped(1, 16, 2, 16, 700, 128, causal=False)),
    ("pack1_L128_full_tile", shaped(1, 4, 2, 128, 600, 128)),
]


SCHEDULES = {"chosen": 0, "split": tb.TFA_DEBUG_FORCE_SPLIT, "whole": tb.TFA_DEBUG_NO_SPLIT}


@pytest.mark.parametrize("schedule", sorted(SCHEDULES))
@pytest.mark.parametrize("name,w", SMALL, ids=[n for n, _ in SMALL])
def test_parity_small(name, w, schedule):
    o, (q, k, v, km) = _run(w, seed=1, flags=SCHEDULES[schedule])
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km)
    err = _assert_close(o, ref, name)
    print(f"{name} [{schedule}]: max abs err {err:.3e}")


def test_fully_masked_rows_are_exact_zeros():
    # tiny-llm Week 2 Day 5, Task 2: 9 query rows, 17 keys, every key masked
    w = shaped(1, 4, 2, 9, 17, 128)
    q, k, v, _ = make_inputs(w, seed=2)
    km = torch.zeros(1, 17)
    o, _ = _run(w, inputs=(q, k, v, km))
    assert torch.all(o == 0).item()
    # partially masked batch: batch 1 has no key at all, batch 0 is ordinary
    w = shaped(2, 4, 2, 40, 90, 128)
    q, k, v, _ = make_inputs(w, seed=3)
    km = torch.ones(2, 90)
    km[1] = 0
    km[0, :30] = 0  # rows whose causal range lies inside the dropped prefix... none (P=50)
    o, _ = _run(w, inputs=(q, k, v, km))
    assert torch.all(o[1] == 0).item()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, key_mask=km)
    _assert_close(o, ref, "partially masked batch")


def test_rows_that_see_no_key_until_late_tiles():
    # window + key mask that empties the first visited tiles of many rows
    w = shaped(1, 4, 2, 300, 900, 128, window=300)
    q, k, v, _ = make_inputs(w, seed=4)
    km = torch.ones(1, 900)
    km[0, 600:800] = 0
    o, _ = _run(w, inputs=(q, k, v, km))
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, window=300, key_mask=km)
    _assert_close(o, ref, "late first key")


@pytest.mark.parametrize("name", ["witness_33x47", "swa_small", "keymask_small", "bidir_small"])
def test_tile_skipping_and_interior_masking_are_bit_exact(name):
    """Skipping unreachable key tiles and skipping the mask on interior tiles
    change nothing, bit for bit (mlx-lm PR 2006: the banded result equals the
    single call exactly)."""
    w = {"witness_33x47": WORKLOADS["witness_33x47"],
         "swa_small": shaped(1, 4, 2, 512, 1023 + 512, 128, window=1024),
         "keymask_small": shaped(1, 4, 2, 300, 800, 128, key_mask_keep=0.9),
         "bidir_small": shaped(1, 4, 2, 200, 400, 128, causal=False)}[name]
    o0, inp = _run(w, seed=5)
    for flags in (tb.TFA_DEBUG_NO_TILE_SKIP, tb.TFA_DEBUG_MASK_ALL,
                  tb.TFA_DEBUG_NO_TILE_SKIP | tb.TFA_DEBUG_MASK_ALL):
        o1, _ = _run(w, inputs=inp, flags=flags)
        assert torch.equal(o0, o1), f"flags {flags} changed the result"


def test_deterministic_and_in_bounds():
    w = shaped(2, 6, 2, 300, 700, 128, window=200)
    q, k, v, _ = make_inputs(w, seed=6)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    pad = 4096
    n = q.numel()
    canary = torch.full((n + 2 * pad,), 1234.0, dtype=torch.bfloat16, device="cuda")
    out = canary[pad:pad + n].view(q.shape)
    tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, window=200, out=out)
    tb.check_status()
    assert torch.all(canary[:pad] == 1234.0).item() and torch.all(canary[pad + n:] == 1234.0).item()
    again = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, window=200)
    tb.check_status()
    assert torch.equal(out, again)


def test_host_entry_matches_device_entry():
    w = shaped(1, 8, 2, 200, 450, 128, key_mask_keep=0.8)
    q, k, v, km = make_inputs(w, seed=7)
    dev, _ = _run(w, inputs=(q, k, v, km))
    host = tb.prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                           scale=w.softmax_scale, causal=True, key_mask=km)
    assert torch.equal(host, dev.cpu())


@pytest.mark.parametrize("name,w,pinned", [
    # three pipeline stages, one batch element each, with a key mask and D = 64
    ("b3_element_stages", shaped(3, 8, 4, 64, 300, 64, key_mask_keep=0.7), True),
    # 20 batch elements: four stages of five whole elements; short rows run packed
    ("b20_batch_stages", shaped(20, 4, 2, 16, 130, 128), True),
    # pageable host memory (copies synchronous to the host, same results); two
    # stages per element over its three KV groups (2 + 1)
    ("pageable_ragged_groups", shaped(2, 6, 3, 150, 400, 128, window=100), False),
])
def test_host_entry_pipelined_stages(name, w, pinned):
    q, k, v, km = make_inputs(w, seed=11)
    dev, _ = _run(w, inputs=(q, k, v, km))
    prep = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    host = tb.prefill_host(prep(q), prep(k), prep(v), scale=w.softmax_scale, causal=w.causal,
                           window=w.window, key_mask=km)
    assert torch.equal(host, dev.cpu()), name


def test_stream_argument_is_respected():
    w = shaped(1, 4, 2, 128, 256, 128)
    q, k, v, _ = make_inputs(w, seed=8)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
        o = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, stream=s)
    s.synchronize()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True)
    _assert_close(o, ref, "side stream")


def _sample_rows(w, n_per_head=24, seed=0):
    """Rows to check at full size: tile edges, tails and random rows, every head."""
    return sample_rows(w, n_per_head=n_per_head, seed=seed)


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items()
                                  if n != "witness_33x47" and w.kind == "dense"])
def test_parity_full_size_sampled(name):
    w = WORKLOADS[name]
    o, (q, k, v, km) = _run(w, seed=0)
    n_per_head = 12 if w.S >= 16384 else 24
    rows = _sample_rows(w, n_per_head=n_per_head)
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km, softcap=w.softcap, sinks=make_sinks(w, 0), rows=rows)
    got = o.reshape(-1, w.D)[torch.as_tensor(rows, device=o.device)]
    err = _assert_close(got, ref, name)
    # properties that hold for every row at any size
    of = o.float()
    assert torch.isfinite(of).all().item()
    print(f"{name}: {rows.size} sampled rows, max abs err {err:.3e}")


@pytest.mark.parametrize("w", [
    shaped(1, 1, 1, 256, 65536, 128, name="one_item_over_every_cta"),
    shaped(1, 2, 1, 300, 40000, 64, window=30000, key_mask_keep=0.95, name="split_d64_window_mask"),
    shaped(2, 4, 2, 1000, 5000, 128, causal=False, k_scale=4.0, name="split_bidirectional"),
], ids=lambda w: w.name)
def test_split_key_ranges_merge_exactly(w):
    """Query tiles whose key range is cut across CTAs and merged (online-softmax
    merge of partial max/sum/accumulator) against the oracle, and against the
    whole-item schedule that never cuts."""
    o, (q, k, v, km) = _run(w, seed=9, flags=tb.TFA_DEBUG_FORCE_SPLIT)
    o_whole, _ = _run(w, inputs=(q, k, v, km), flags=tb.TFA_DEBUG_NO_SPLIT)
    rows = _sample_rows(w, n_per_head=min(w.L, 64))
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km, rows=rows)
    idx = torch.as_tensor(rows, device=o.device)
    _assert_close(o.reshape(-1, w.D)[idx], ref, w.name + " split")
    _assert_close(o_whole.reshape(-1, w.D)[idx], ref, w.name + " whole items")
    _assert_close(o.float().cpu().double().numpy(), o_whole.float().cpu().double().numpy(),
                  w.name + " split vs whole")
