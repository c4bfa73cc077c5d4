"""Pins for the fp64 CPU oracle: checks against what the pages and the
mathematics fix, independent of the oracle's own code.

Each pin takes an attention callable with the oracle's signature, so the same
pins run against mutants of the oracle (planted mistakes), which must fail at
least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).bfloat16()


def _one_hot_values(B, Hkv, S, D):
    """V[b,g,j,:] = e_j so that attention with q = 0 returns the uniform
    distribution over the allowed keys in its first S coordinates."""
    assert D >= S
    v = torch.zeros(B, Hkv, S, D)
    for j in range(S):
        v[:, :, j, j] = 1.0
    return v.bfloat16()


def _visibility_via_attention(attn, L, S, causal, window, key_mask=None):
    D = max(8, S)
    q = torch.zeros(1, 1, L, D).bfloat16()
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(3)).bfloat16()
    v = _one_hot_values(1, 1, S, D)
    o = attn(q, k, v, scale=1.0, causal=causal, window=window, key_mask=key_mask)
    return o[0, 0, :, :S] > 0.0, o[0, 0, :, :S]


# ---------------------------------------------------------------------------
# pins: each raises AssertionError when the attention callable is wrong
# ---------------------------------------------------------------------------

def pin_golden_visibility(attn):
    for name in ["visibility_L3_S7_causal.txt", "visibility_window_L4_S6_W3.txt",
                 "visibility_window_L3_S3_W1.txt"]:
        g = _read_golden(name)
        L, S, causal, window = map(int, g[0])
        vis, probs = _visibility_via_attention(attn, L, S, bool(causal), window)
        for i, (lo, hi) in enumerate(g[1:]):
            expect = np.zeros(S, dtype=bool)
            expect[int(lo):int(hi) + 1] = True
            assert np.array_equal(vis[i], expect), (name, i, vis[i], expect)
            # uniform weights over exactly the visible keys
            assert np.allclose(probs[i][expect], 1.0 / expect.sum(), atol=1e-12), (name, i)


def pin_fully_masked_rows_are_zero(attn):
    g = _read_golden("fully_masked_9x17.txt")
    L, S = map(int, g[0])
    value = float(g[1][0])
    w = shaped(1, 4, 2, L, S, 16)
    q, k, v, _ = make_inputs(w, seed=5)
    km = torch.zeros(1, S)
    o = attn(q, k, v, scale=0.25, causal=True, window=0, key_mask=km)
    assert np.all(np.isfinite(o))
    assert np.all(o == value)
    # bidirectional too
    o = attn(q, k, v, scale=0.25, causal=False, window=0, key_mask=km)
    assert np.all(o == value)


def pin_all_ones_mask_equals_no_mask(attn):
    w = shaped(2, 4, 2, 13, 29, 16)
    q, k, v, _ = make_inputs(w, seed=6)
    for causal, window in [(True, 0), (True, 5), (False, 0)]:
        a = attn(q, k, v, scale=0.25, causal=causal, window=window, key_mask=torch.ones(2, 29))
        b = attn(q, k, v, scale=0.25, causal=causal, window=window, key_mask=None)
        assert np.array_equal(a, b)


def pin_gqa_equals_replicated_mha(attn):
    w = shaped(2, 6, 2, 11, 19, 16)
    q, k, v, _ = make_inputs(w, seed=7)
    G = 3
    k_rep = k.repeat_interleave(G, dim=1)
    v_rep = v.repeat_interleave(G, dim=1)
    for causal, window in [(True, 0), (True, 4), (False, 0)]:
        a = attn(q, k, v, scale=0.3, causal=causal, window=window)
        b = attn(q, k_rep, v_rep, scale=0.3, causal=causal, window=window)
        assert np.allclose(a, b, atol=1e-13, rtol=0)


def _sdpa_reference(q, k, v, scale, allowed):
    """torch's own scaled_dot_product_attention in float64 on CPU (GQA mode)."""
    out = F.scaled_dot_product_attention(q.double(), k.double(), v.double(), attn_mask=allowed,
                                         scale=scale, enable_gqa=True)
    return out.numpy()


def pin_matches_torch_sdpa(attn):
    # causal masks built the way tinygrad's symbolic prefill builds them:
    # full(-inf).triu(start_pos + 1) over (T, start_pos + T), i.e. allowed = tril(start_pos)
    for (B, Hq, Hkv, L, S, D, scale) in [(1, 8, 2, 33, 47, 128, 1 / math.sqrt(128)),
                                         (2, 4, 4, 9, 9, 64, 0.125),
                                         (1, 6, 3, 5, 40, 32, 0.37)]:
        q, k, v, _ = make_inputs(shaped(B, Hq, Hkv, L, S, D), seed=11)
        P = S - L
        allowed = torch.ones(L, S, dtype=torch.bool).tril(diagonal=P)
        ref = _sdpa_reference(q, k, v, scale, allowed)
        got = attn(q, k, v, scale=scale, causal=True, window=0)
        assert np.allclose(got, ref, atol=1e-12, rtol=1e-10), (B, Hq, L, S)
        ref = _sdpa_reference(q, k, v, scale, torch.ones(L, S, dtype=torch.bool))
        got = attn(q, k, v, scale=scale, causal=False, window=0)
        assert np.allclose(got, ref, atol=1e-12, rtol=1e-10)
    # sliding window as a band: tril(P) minus tril(P - W)
    B, Hq, Hkv, L, S, D, W = 1, 4, 2, 20, 35, 32, 6
    q, k, v, _ = make_inputs(shaped(B, Hq, Hkv, L, S, D), seed=12)
    P = S - L
    band = torch.ones(L, S, dtype=torch.bool).tril(diagonal=P) & \
        ~torch.ones(L, S, dtype=torch.bool).tril(diagonal=P - W)
    ref = _sdpa_reference(q, k, v, 0.2, band)
    got = attn(q, k, v, scale=0.2, causal=True, window=W)
    assert np.allclose(got, ref, atol=1e-12, rtol=1e-10)
    # key mask: per-batch boolean row broadcast over heads and queries
    B, Hq, Hkv, L, S, D = 2, 4, 2, 12, 30, 32
    q, k, v, km = make_inputs(shaped(B, Hq, Hkv, L, S, D, key_mask_keep=0.7), seed=13)
    P = S - L
    allowed = torch.ones(L, S, dtype=torch.bool).tril(diagonal=P)[None, None] & (km > 0.5)[:, None, None, :]
    live = allowed.any(-1)  # rows with at least one allowed key (SDPA gives NaN otherwise)
    ref = _sdpa_reference(q, k, v, 0.2, allowed)
    got = attn(q, k, v, scale=0.2, causal=True, window=0, key_mask=km)
    livemask = live.expand(B, Hq, L).numpy()
    assert np.allclose(got[livemask], ref[livemask], atol=1e-12, rtol=1e-10)
    assert np.all(got[~livemask] == 0.0)


def pin_constant_values_give_constant_rows(attn):
    w = shaped(1, 4, 2, 10, 24, 16)
    q, k, _, _ = make_inputs(w, seed=8)
    c = torch.linspace(-2, 2, 16)
    v = c.expand(1, 2, 24, 16).contiguous().bfloat16()
    o = attn(q, k, v, scale=0.5, causal=True, window=7)
    assert np.allclose(o, v[0, 0, 0].double().numpy()[None, None, None, :], atol=1e-13)


def pin_window_one_returns_own_value(attn):
    w = shaped(1, 4, 2, 9, 17, 16)
    q, k, v, _ = make_inputs(w, seed=9)
    o = attn(q, k, v, scale=0.25, causal=True, window=1)
    P = 17 - 9
    for h in range(4):
        g = h // 2
        assert np.array_equal(o[0, h], v[0, g, P:P + 9].double().numpy())


def pin_wide_window_equals_causal(attn):
    w = shaped(1, 4, 2, 12, 31, 16)
    q, k, v, _ = make_inputs(w, seed=10)
    base = attn(q, k, v, scale=0.25, causal=True, window=0)
    for W in [31, 32, 1000]:
        assert np.array_equal(attn(q, k, v, scale=0.25, causal=True, window=W), base)
    assert not np.allclose(attn(q, k, v, scale=0.25, causal=True, window=30), base)


def pin_chunked_prefix_invariance(attn):
    """A chunk of L rows after a prefix equals the last L rows of the full causal
    run over the same keys (tinygrad's split-prefix prefill test idea)."""
    Sfull, L = 40, 13
    w = shaped(1, 4, 2, Sfull, Sfull, 16)
    q, k, v, _ = make_inputs(w, seed=14)
    full = attn(q, k, v, scale=0.25, causal=True, window=0)
    chunk = attn(q[:, :, Sfull - L:].contiguous(), k, v, scale=0.25, causal=True, window=0)
    assert np.allclose(chunk, full[:, :, Sfull - L:], atol=1e-14, rtol=0)
    fullw = attn(q, k, v, scale=0.25, causal=True, window=5)
    chunkw = attn(q[:, :, Sfull - L:].contiguous(), k, v, scale=0.25, causal=True, window=5)
    assert np.allclose(chunkw, fullw[:, :, Sfull - L:], atol=1e-14, rtol=0)


def pin_softcap_acts_after_the_scale(attn):
    """brotensor flash_attention.h, Gemma-2 extensions: the cap applies to the
    scaled score.  Doubling q (exact in bf16) while halving the scale leaves
    every scaled score, hence the output, unchanged; a cap taken before the
    scale would not be invariant.  A small cap must also change the result."""
    w = shaped(1, 4, 2, 12, 40, 32, k_scale=4.0)
    q, k, v, _ = make_inputs(w, seed=31)
    for cap in (2.0, 7.5):
        a = attn(q, k, v, scale=0.3, causal=True, window=0, softcap=cap)
        b = attn((q.float() * 2).bfloat16(), k, v, scale=0.15, causal=True, window=0, softcap=cap)
        assert np.allclose(a, b, atol=1e-13, rtol=0)
        assert not np.allclose(a, attn(q, k, v, scale=0.3, causal=True, window=0), atol=1e-3)


def pin_softcap_limits(attn):
    """tanh(x) -> x as the cap grows: a huge cap is no cap.  As the cap shrinks
    every score goes to 0 and the weights to uniform: the output becomes the
    plain mean of the visible values.  One visible key still returns its value."""
    w = shaped(1, 4, 2, 10, 30, 16, k_scale=4.0)
    q, k, v, _ = make_inputs(w, seed=32)
    base = attn(q, k, v, scale=0.25, causal=True, window=0)
    assert np.allclose(attn(q, k, v, scale=0.25, causal=True, window=0, softcap=1e9), base,
                       atol=1e-12, rtol=0)
    tiny = attn(q, k, v, scale=0.25, causal=False, window=0, softcap=1e-12)
    mean = v.double().mean(dim=2).numpy()  # [B, Hkv, D]
    for h in range(4):
        assert np.allclose(tiny[0, h], mean[0, h // 2][None, :], atol=1e-10)
    one = attn(q, k, v, scale=0.25, causal=True, window=1, softcap=3.0)
    for h in range(4):
        assert np.array_equal(one[0, h], v[0, h // 2, 20:30].double().numpy())


def pin_sinks_match_sdpa_with_a_null_key(attn):
    """A sink is a logit with no value row: torch's SDPA (fp64) over the keys
    plus one all-zero key and value, whose additive mask entry is the sink
    logit, gives the same output -- rows with no visible key included (their
    only mass is the sink's, times a zero value)."""
    B, Hq, Hkv, L, S, D, W = 2, 6, 2, 11, 37, 32, 9
    q, k, v, km = make_inputs(shaped(B, Hq, Hkv, L, S, D, key_mask_keep=0.6), seed=33)
    sinks = torch.tensor([-1.5, 0.0, 0.7, 2.5, -30.0, 6.0], dtype=torch.float32)
    km[1, :] = 0.0  # batch 1: every row fully masked
    P = S - L
    for window in (0, W):
        allowed = torch.ones(L, S, dtype=torch.bool).tril(diagonal=P)
        if window:
            allowed &= ~torch.ones(L, S, dtype=torch.bool).tril(diagonal=P - window)
        allowed = allowed[None, None] & (km > 0.5)[:, None, None, :]
        bias = torch.zeros(B, Hq, L, S + 1, dtype=torch.float64)
        bias[..., :S] = torch.where(allowed, 0.0, -math.inf)
        bias[..., S] = sinks.double()[None, :, None]
        kz = torch.cat([k.double(), torch.zeros(B, Hkv, 1, D, dtype=torch.float64)], dim=2)
        vz = torch.cat([v.double(), torch.zeros(B, Hkv, 1, D, dtype=torch.float64)], dim=2)
        ref = F.scaled_dot_product_attention(q.double(), kz, vz, attn_mask=bias, scale=0.2,
                                             enable_gqa=True).numpy()
        got = attn(q, k, v, scale=0.2, causal=True, window=window, key_mask=km, sinks=sinks)
        assert np.allclose(got, ref, atol=1e-12, rtol=1e-10)
        assert np.all(got[1] == 0.0)
    none = attn(q, k, v, scale=0.2, causal=True, window=0, key_mask=km)
    neg = attn(q, k, v, scale=0.2, causal=True, window=0, key_mask=km,
               sinks=torch.full((Hq,), -math.inf))
    assert np.array_equal(none, neg)


ATTENTION_PINS = [
    pin_golden_visibility,
    pin_fully_masked_rows_are_zero,
    pin_all_ones_mask_equals_no_mask,
    pin_gqa_equals_replicated_mha,
    pin_matches_torch_sdpa,
    pin_constant_values_give_constant_rows,
    pin_window_one_returns_own_value,
    pin_wide_window_equals_causal,
    pin_chunked_prefix_invariance,
    pin_softcap_acts_after_the_scale,
    pin_softcap_limits,
    pin_sinks_match_sdpa_with_a_null_key,
]


@pytest.mark.parametrize("pin", ATTENTION_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.attention)


@pytest.mark.parametrize("mutation", sorted(oracle.MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation):
    def mutant(q, k, v, **kw):
        return oracle.attention_mutant(q, k, v, mutation=mutation, **kw)

    caught = []
    for pin in ATTENTION_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutation {mutation} passed every pin"


# ---------------------------------------------------------------------------
# pins on the oracle's other entry points
# ---------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_vanish_off_mask():
    w = shaped(2, 4, 2, 17, 41, 32, key_mask_keep=0.8)
    q, k, _, km = make_inputs(w, seed=15)
    for causal, window in [(True, 0), (True, 9), (False, 0)]:
        for b, h in [(0, 0), (1, 3)]:
            Wt = oracle.softmax_weights(q, k, b=b, h=h, scale=0.2, causal=causal, window=window,
                                        key_mask=km)
            vis = oracle.visibility(17, 41, causal=causal, window=window, key_mask_row=km[b])
            sums = Wt.sum(1)
            live = vis.any(1)
            assert np.allclose(sums[live], 1.0, atol=1e-14)
            assert np.all(sums[~live] == 0.0)
            assert np.all(Wt[~vis] == 0.0)
            assert np.all(Wt[vis] > 0.0)


def test_witness_pair_count_matches_golden():
    g = _read_golden("witness_pairs.txt")
    L, S, Hq = map(int, g[0])
    per_head, total = int(g[1][0]), int(g[2][0])
    assert oracle.count_pairs(1, 1, L, S, causal=True) == per_head
    assert oracle.count_pairs(1, Hq, L, S, causal=True) == total


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_pair_count_closed_form(name):
    w = WORKLOADS[name]
    L, S, P, W = w.L, w.S, w.S - w.L, w.window
    if not w.causal:
        closed = L * S
    elif W <= 0:
        closed = L * P + L * (L + 1) // 2           # sum_i (P + i + 1)
    else:
        closed = sum(min(W, P + i + 1) for i in range(L))
    closed *= w.B * w.Hq
    assert oracle.count_pairs(w.B, w.Hq, L, S, causal=w.causal, window=W) == closed
    if w.key_mask_keep is not None:
        # with the key mask: key j is counted once for every row that reaches it
        km = make_inputs(w.with_(Hq=1, Hkv=1, D=8), seed=0)[3]
        reach = np.array([L - max(0, j - P) for j in range(S)], dtype=np.int64)
        with_mask = int(((km.numpy() > 0.5).astype(np.int64) * reach).sum()) * w.Hq
        assert oracle.count_pairs(w.B, w.Hq, L, S, causal=True, window=0,
                                  key_mask=km) == with_mask


def test_blockwise_online_softmax_matches_plain():
    """The tile-by-tile merge with masked-tile skipping gives the plain result."""
    cases = [
        (shaped(1, 8, 2, 33, 47, 32), dict(causal=True, window=0)),
        (shaped(1, 4, 2, 40, 71, 16), dict(causal=True, window=9)),
        (shaped(2, 4, 1, 20, 20, 16), dict(causal=False, window=0)),
        (shaped(2, 4, 2, 24, 50, 16, key_mask_keep=0.6), dict(causal=True, window=0)),
    ]
    for w, kw in cases:
        q, k, v, km = make_inputs(w, seed=16)
        plain = oracle.attention(q, k, v, scale=0.3, key_mask=km, **kw)
        for bq, bk in [(16, 16), (128, 128), (8, 5)]:
            tiled, visited = oracle.attention_blockwise(q, k, v, scale=0.3, key_mask=km, bq=bq,
                                                        bk=bk, skip_empty=True, **kw)
            assert np.allclose(tiled, plain, atol=1e-12, rtol=1e-12), (w, bq, bk)
            dense, all_tiles = oracle.attention_blockwise(q, k, v, scale=0.3, key_mask=km, bq=bq,
                                                          bk=bk, skip_empty=False, **kw)
            assert np.allclose(dense, plain, atol=1e-12, rtol=1e-12)
            assert visited <= all_tiles


def test_sliding_window_skips_tiles():
    """With a 1024-key window over a rotating cache most key tiles are skipped."""
    w = shaped(1, 1, 1, 256, 1023 + 256, 8)
    q, k, v, _ = make_inputs(w, seed=17)
    _, visited = oracle.attention_blockwise(q, k, v, scale=0.3, causal=True, window=1024, bq=128,
                                            bk=128, skip_empty=True)
    _, dense = oracle.attention_blockwise(q, k, v, scale=0.3, causal=True, window=1024, bq=128,
                                          bk=128, skip_empty=False)
    assert visited < dense


def test_row_subset_matches_full():
    w = shaped(2, 4, 2, 19, 30, 16, key_mask_keep=0.8)
    q, k, v, km = make_inputs(w, seed=18)
    full = oracle.attention(q, k, v, scale=0.3, causal=True, window=7, key_mask=km)
    rows = np.array([0, 5, 18, 19, 77, 2 * 4 * 19 - 1])
    sub = oracle.attention(q, k, v, scale=0.3, causal=True, window=7, key_mask=km, rows=rows)
    assert np.array_equal(sub, full.reshape(-1, 16)[rows])


def test_oracle_rejects_bad_arguments():
    q, k, v, _ = make_inputs(shaped(1, 3, 2, 4, 8, 8), seed=0)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, scale=1.0, causal=True)  # 3 % 2 != 0
