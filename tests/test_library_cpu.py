"""CPU-side checks of the CUDA library: it loads, exports every declared entry
point, rejects bad arguments before touching the GPU, and its work
enumeration (the tile scheduler's host view) is exact against the oracle's
visibility rule.  No compute call runs here."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.flops import allowed_pairs
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped


def test_library_exports_every_declared_symbol():
    names = tb.declared_symbols()
    assert {"tfa_prefill", "tfa_prefill_debug", "tfa_prefill_host", "tfa_check_status",
            "tfa_status_string", "tfa_plan_qtile"} <= set(names)
    lib = tb.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code in range(16):
        s = tb.status_string(code)
        assert s and s != "unknown status"
    assert tb.status_string(99) == "unknown status"


# pointers that are never dereferenced: validation fails before any CUDA call
A16 = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10008)


def _call(**over):
    a = dict(q=A16, k=A16, v=A16, o=A16, B=1, Hq=8, Hkv=2, L=33, S=47, D=128, scale=0.088,
             causal=1, window=0, key_mask=None, stream=None)
    a.update(over)
    return tb.tfa_prefill(**a)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), tb.TFA_ERR_NULL),
    (dict(o=None), tb.TFA_ERR_NULL),
    (dict(Hq=7, Hkv=2), tb.TFA_ERR_HEADS),
    (dict(Hkv=0), tb.TFA_ERR_HEADS),
    (dict(L=8, S=47), tb.TFA_ERR_SHORT_QUERY),
    (dict(L=1, S=1), tb.TFA_ERR_SHORT_QUERY),
    (dict(B=0), tb.TFA_ERR_SHAPE),
    (dict(L=33, S=32), tb.TFA_ERR_SHAPE),
    (dict(D=96), tb.TFA_ERR_HEAD_DIM),
    (dict(D=256), tb.TFA_ERR_HEAD_DIM),
    (dict(causal=0, window=16), tb.TFA_ERR_WINDOW),
    (dict(q=MIS), tb.TFA_ERR_ALIGN),
    (dict(v=MIS), tb.TFA_ERR_ALIGN),
    (dict(key_mask=ctypes.c_void_p(0x10002)), tb.TFA_ERR_ALIGN),
    (dict(scale=float("nan")), tb.TFA_ERR_SCALE),
    (dict(scale=float("inf")), tb.TFA_ERR_SCALE),
])
def test_rejections_happen_before_launch(over, code):
    assert _call(**over) == code


def _call_ex(**over):
    a = dict(q=A16, k=A16, v=A16, o=A16, B=1, Hq=8, Hkv=2, L=33, S=47, D=128, scale=0.088,
             causal=1, window=0, key_mask=None, softcap=0.0, sinks=None, stream=None)
    a.update(over)
    return tb.tfa_attention_ex(**a)


@pytest.mark.parametrize("over,code", [
    (dict(softcap=-1.0), tb.TFA_ERR_SOFTCAP),
    (dict(softcap=float("nan")), tb.TFA_ERR_SOFTCAP),
    (dict(softcap=float("inf")), tb.TFA_ERR_SOFTCAP),
    (dict(softcap=30.0, scale=0.0), tb.TFA_ERR_SOFTCAP),
    (dict(sinks=ctypes.c_void_p(0x10002)), tb.TFA_ERR_ALIGN),
    (dict(L=0, S=47), tb.TFA_ERR_SHORT_QUERY),
    (dict(L=1, S=0), tb.TFA_ERR_SHAPE),
    (dict(Hq=7, Hkv=2, softcap=30.0), tb.TFA_ERR_HEADS),
    (dict(causal=0, window=4, L=3), tb.TFA_ERR_WINDOW),
    (dict(D=80, L=1), tb.TFA_ERR_HEAD_DIM),
])
def test_score_variant_rejections_happen_before_launch(over, code):
    assert _call_ex(**over) == code


def test_ring_rejections_happen_before_launch():
    a = dict(q=A16, k=A16, v=A16, o=A16, B=1, Hq=8, Hkv=2, L=33, S=5000, ring_rows=1088, D=128,
             scale=0.088, window=1024, softcap=0.0, sinks=None, stream=None)
    assert tb.tfa_prefill_ring(**{**a, "window": 0}) == tb.TFA_ERR_RING
    assert tb.tfa_prefill_ring(**{**a, "ring_rows": 1000}) == tb.TFA_ERR_RING   # not a multiple of 64
    assert tb.tfa_prefill_ring(**{**a, "ring_rows": 1024}) == tb.TFA_ERR_RING   # < 1023 + 33
    assert tb.tfa_prefill_ring(**{**a, "S": 20}) == tb.TFA_ERR_SHAPE            # S < L
    assert tb.tfa_prefill_ring(**{**a, "Hq": 7}) == tb.TFA_ERR_HEADS
    assert tb.tfa_prefill_ring(**{**a, "softcap": -2.0}) == tb.TFA_ERR_SOFTCAP
    assert tb.tfa_prefill_ring(**{**a, "k": MIS}) == tb.TFA_ERR_ALIGN


def test_varlen_rejections_happen_before_launch():
    a = dict(q=A16, k=A16, v=A16, o=A16, cu_q=A16, cu_k=A16, B=3, Hq=8, Hkv=2, total_q=100,
             total_k=300, max_seqlen_q=60, D=128, scale=0.088, causal=1, window=0, softcap=0.0,
             sinks=None, stream=None)
    assert tb.tfa_prefill_varlen(**{**a, "total_q": 0, "q": None}) == tb.TFA_OK  # nothing to do
    assert tb.tfa_prefill_varlen(**{**a, "cu_k": None}) == tb.TFA_ERR_NULL
    assert tb.tfa_prefill_varlen(**{**a, "Hkv": 3}) == tb.TFA_ERR_HEADS
    assert tb.tfa_prefill_varlen(**{**a, "B": 0}) == tb.TFA_ERR_SHAPE
    assert tb.tfa_prefill_varlen(**{**a, "B": tb.MAX_VARLEN_SEQS + 1}) == tb.TFA_ERR_SHAPE
    assert tb.tfa_prefill_varlen(**{**a, "max_seqlen_q": 0}) == tb.TFA_ERR_SHAPE
    assert tb.tfa_prefill_varlen(**{**a, "total_k": 0}) == tb.TFA_ERR_SHAPE
    assert tb.tfa_prefill_varlen(**{**a, "D": 96}) == tb.TFA_ERR_HEAD_DIM
    assert tb.tfa_prefill_varlen(**{**a, "causal": 0, "window": 5}) == tb.TFA_ERR_WINDOW
    assert tb.tfa_prefill_varlen(**{**a, "cu_q": ctypes.c_void_p(0x10002)}) == tb.TFA_ERR_ALIGN
    assert tb.tfa_prefill_varlen(**{**a, "scale": float("nan")}) == tb.TFA_ERR_SCALE
    assert tb.tfa_prefill_varlen(**{**a, "softcap": float("inf")}) == tb.TFA_ERR_SOFTCAP


def test_debug_rejects_unknown_flags_before_launch():
    assert tb.tfa_prefill_debug(A16, A16, A16, A16, 1, 8, 2, 33, 47, 128, 0.1, 1, 0, None, None,
                                64) == tb.TFA_ERR_FLAGS


def test_host_entry_validates_first():
    assert tb.tfa_prefill_host(A16, A16, A16, A16, 1, 6, 4, 33, 47, 128, 0.1, 1, 0, None,
                               None) == tb.TFA_ERR_HEADS


def _plan_cases():
    cases = []
    for name, w in WORKLOADS.items():
        if w.L * w.S <= 2048 * 8192:
            cases.append((name, w.L, w.S, w.causal, w.window, w.key_mask_keep is not None))
    cases += [("ragged", 300, 301, True, 0, False), ("tiny", 9, 9, True, 0, False),
              ("win1", 130, 700, True, 1, False), ("win129", 257, 1000, True, 129, False),
              ("bidir_ragged", 200, 333, False, 0, False), ("wide", 200, 333, True, 5000, False),
              ("w127", 383, 1111, True, 127, False)]
    return cases


@pytest.mark.parametrize("case", _plan_cases(), ids=lambda c: c[0])
def test_tile_enumeration_is_exact(case):
    """Every allowed (row, key) pair lies in a visited key tile; the first and
    last visited tiles each hold an allowed pair (nothing reachable is skipped,
    nothing skipped is reachable); tiles marked interior need no mask for any
    valid row."""
    _, L, S, causal, window, has_km = case
    P = S - L
    nqt = (L + 127) // 128
    for qt in range(nqt):
        rc, lo, hi, needs = tb.tfa_plan_qtile(L, S, causal, window, has_km, qt)
        assert rc == 0
        r0, r1 = qt * 128, min(qt * 128 + 128, L)
        rows = np.arange(r0, r1)[:, None]
        keys = np.arange(S)[None, :]
        pos = P + rows
        allowed = np.ones((r1 - r0, S), dtype=bool)
        if causal:
            allowed &= keys <= pos
            if window > 0:
                allowed &= keys > pos - window
        tiles = np.nonzero(allowed.any(0))[0] // 128
        assert tiles.min() == lo and tiles.max() == hi
        for j in range(lo, hi + 1):
            blk = allowed[:, j * 128:min(j * 128 + 128, S)]
            full = blk.shape[1] == 128 and blk.all()
            if not needs[j - lo]:
                assert full, (qt, j)
            if has_km:
                assert needs[j - lo]
    # the same rule, counted by the oracle's brute force, for small cases
    if L * S <= 400 * 1200:
        assert allowed_pairs(1, 1, L, S, causal=causal, window=window) == \
            oracle.count_pairs(1, 1, L, S, causal=causal, window=window)


def test_visibility_rule_matches_oracle_on_small_shapes():
    for L, S, causal, window in [(9, 9, True, 0), (10, 40, True, 3), (12, 30, False, 0),
                                 (33, 47, True, 0), (20, 25, True, 1)]:
        vis = oracle.visibility(L, S, causal=causal, window=window)
        P = S - L
        rows = np.arange(L)[:, None] + P
        keys = np.arange(S)[None, :]
        mine = np.ones((L, S), dtype=bool)
        if causal:
            mine &= keys <= rows
            if window > 0:
                mine &= keys > rows - window
        assert np.array_equal(vis, mine)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_flop_count_matches_oracle_count(name):
    w = WORKLOADS[name]
    km = None
    if w.key_mask_keep is not None:
        km = make_inputs(w.with_(Hq=1, Hkv=1, D=8), seed=0)[3]
    assert allowed_pairs(w.B, w.Hq, w.L, w.S, causal=w.causal, window=w.window, key_mask=km) == \
        oracle.count_pairs(w.B, w.Hq, w.L, w.S, causal=w.causal, window=w.window, key_mask=km)


def test_flop_count_small_key_mask_cases():
    for (B, L, S, causal, window) in [(2, 10, 30, True, 0), (3, 9, 9, True, 4), (2, 12, 20, False, 0)]:
        km = (torch.rand(B, S, generator=torch.Generator().manual_seed(1)) > 0.3).float()
        assert allowed_pairs(B, 3, L, S, causal=causal, window=window, key_mask=km) == \
            oracle.count_pairs(B, 3, L, S, causal=causal, window=window, key_mask=km)


@pytest.mark.parametrize("L,code", [(0, tb.TFA_ERR_SHAPE), (9, tb.TFA_ERR_SHAPE),
                                    (64, tb.TFA_ERR_SHAPE)])
def test_decode_accepts_only_short_queries(L, code):
    assert tb.tfa_decode(A16, A16, A16, A16, 1, 8, 2, L, 100, 128, 0.1, 1, 0, None, None) == code


def test_decode_validates_like_prefill():
    assert tb.tfa_decode(None, A16, A16, A16, 1, 8, 2, 1, 100, 128, 0.1, 1, 0, None,
                         None) == tb.TFA_ERR_NULL
    assert tb.tfa_decode(A16, A16, A16, A16, 1, 8, 3, 1, 100, 128, 0.1, 1, 0, None,
                         None) == tb.TFA_ERR_HEADS
    assert tb.tfa_decode(A16, A16, A16, A16, 1, 8, 2, 4, 3, 128, 0.1, 1, 0, None,
                         None) == tb.TFA_ERR_SHAPE
    assert tb.tfa_decode(A16, A16, A16, A16, 1, 8, 2, 1, 100, 128, 0.1, 0, 16, None,
                         None) == tb.TFA_ERR_WINDOW


@pytest.mark.parametrize("case", _plan_cases(), ids=lambda c: c[0])
def test_key_tile_enumeration_is_exact(case):
    """The backward pass's view: every allowed (row, key) pair has its row's
    query tile inside the range of its key's tile, and the first and last
    query tiles of each range hold an allowed pair."""
    _, L, S, causal, window, _ = case
    P = S - L
    nkt = (S + 127) // 128
    rows = np.arange(L)[:, None]
    keys = np.arange(S)[None, :]
    allowed = np.ones((L, S), dtype=bool)
    if causal:
        allowed &= keys <= P + rows
        if window > 0:
            allowed &= keys > P + rows - window
    for kt in range(nkt):
        rc, lo, hi = tb.tfa_plan_ktile(L, S, causal, window, kt)
        assert rc == 0
        blk = allowed[:, kt * 128:(kt + 1) * 128].any(axis=1)
        qts = sorted(set(np.nonzero(blk)[0] // 128))
        if not qts:
            assert hi < lo
        else:
            assert (lo, hi) == (qts[0], qts[-1]), (kt, lo, hi, qts[0], qts[-1])


def test_lse_and_saved_backward_reject_before_launch():
    L_ = tb.lib()
    i = (1, 8, 2, 64, 200, 128)
    # forward with log-sum-exp: NULL or misaligned lse, then tfa_prefill's own checks
    assert L_.tfa_prefill_lse(A16, A16, A16, A16, None, *i, 0.1, 1, 0, None, None) == tb.TFA_ERR_NULL
    assert L_.tfa_prefill_lse(A16, A16, A16, A16, ctypes.c_void_p(0x10002), *i, 0.1, 1, 0, None,
                              None) == tb.TFA_ERR_ALIGN
    assert L_.tfa_prefill_lse(A16, A16, A16, A16, A16, 1, 8, 3, 64, 200, 128, 0.1, 1, 0, None,
                              None) == tb.TFA_ERR_HEADS
    # backward from saved statistics: NULL o / lse / gradient, misaligned o or lse
    args = [A16] * 9
    for n, code in ((3, tb.TFA_ERR_NULL), (4, tb.TFA_ERR_NULL), (8, tb.TFA_ERR_NULL)):
        bad = list(args)
        bad[n] = None
        assert L_.tfa_prefill_backward_saved(*bad, *i, 0.1, 1, 0, None, None) == code
    for n, p in ((3, MIS), (4, ctypes.c_void_p(0x10002))):
        bad = list(args)
        bad[n] = p
        assert L_.tfa_prefill_backward_saved(*bad, *i, 0.1, 1, 0, None, None) == tb.TFA_ERR_ALIGN
    assert L_.tfa_prefill_backward_saved(*args, 1, 8, 2, 64, 200, 96, 0.1, 1, 0, None,
                                         None) == tb.TFA_ERR_HEAD_DIM
