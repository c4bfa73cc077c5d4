"""Pins for the oracle's rotating-cache and packed variable-length entry points,
each against the dense oracle (itself pinned in test_oracle_pins.py) on data
rearranged by plain tensor indexing in the test -- an independent construction
of what the two addressing modes must compute -- plus the rules the pages state
(brotensor's varlen causal rule for equal lengths; no cross-sequence
attention).  Planted mistakes must fail at least one pin."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped


# --------------------------------------------------------------- rotating cache

def _ring_from_dense(k_full, R, seed):
    """Ring buffer [B,H,R,D] holding positions [S-R, S) of k_full at row j mod R;
    rows for positions that fell out of the ring are junk."""
    B, H, S, D = k_full.shape
    g = torch.Generator().manual_seed(seed)
    ring = (7.0 * torch.randn(B, H, R, D, generator=g)).bfloat16()
    for j in range(max(0, S - R), S):
        ring[:, :, j % R] = k_full[:, :, j]
    return ring


RING_CASES = [  # (B, Hq, Hkv, L, S, R, W, D)
    (2, 4, 2, 10, 40, 16, 6, 16),    # wrapped twice, prefix 30
    (1, 6, 3, 7, 23, 64, 20, 32),    # ring not yet full (S <= R)
    (1, 4, 1, 9, 77, 17, 9, 16),     # R = W - 1 + L exactly
    (1, 2, 2, 1, 1000, 64, 50, 16),  # one new row (decode)
]


def pin_ring_equals_dense_over_positions(ring_attn):
    for (B, Hq, Hkv, L, S, R, W, D) in RING_CASES:
        q, k, v, _ = make_inputs(shaped(B, Hq, Hkv, L, S, D, k_scale=2.0), seed=R + S)
        kr, vr = _ring_from_dense(k, R, 1), _ring_from_dense(v, R, 2)
        sinks = torch.linspace(-1.0, 1.0, Hq)
        for softcap, sk in [(0.0, None), (3.0, sinks)]:
            got = ring_attn(q, kr, vr, S=S, scale=0.3, window=W, softcap=softcap, sinks=sk)
            ref = oracle.attention(q, k, v, scale=0.3, causal=True, window=W, softcap=softcap,
                                   sinks=sk)
            assert np.array_equal(got, ref), (B, Hq, L, S, R, W)


def test_ring_pin():
    pin_ring_equals_dense_over_positions(oracle.attention_ring)


@pytest.mark.parametrize("mutation", sorted(oracle.RING_MUTATIONS))
def test_ring_planted_mistake_fails(mutation):
    def mutant(*a, **kw):
        return oracle.attention_ring(*a, mutation=mutation, **kw)
    with pytest.raises(AssertionError):
        pin_ring_equals_dense_over_positions(mutant)


def test_ring_rejects_a_ring_too_small_for_the_window():
    q, k, v, _ = make_inputs(shaped(1, 2, 2, 10, 40, 16), seed=1)
    kr = _ring_from_dense(k, 14, 1)
    with pytest.raises(ValueError):
        oracle.attention_ring(q, kr, kr, S=40, scale=0.3, window=6)  # needs R >= 15
    with pytest.raises(ValueError):
        oracle.attention_ring(q, kr, kr, S=40, scale=0.3, window=0)  # ring needs a window


# ---------------------------------------------------- packed variable lengths

def _pack(seqs):
    """seqs: list of [1,H,len,D] tensors -> packed [T,H,D] and int32 prefix sums."""
    parts = [s[0].transpose(0, 1) for s in seqs]  # [len, H, D]
    cu = np.concatenate([[0], np.cumsum([p.shape[0] for p in parts])]).astype(np.int32)
    return torch.cat(parts, dim=0).contiguous(), cu


def _varlen_case(lengths, Hq, Hkv, D, seed, k_scale=1.0):
    qs, ks, vs = [], [], []
    for n, (Lb, Sb) in enumerate(lengths):
        q, k, v, _ = make_inputs(shaped(1, Hq, Hkv, max(Lb, 1), max(Sb, 1), D, k_scale=k_scale),
                                 seed=seed + n)
        qs.append(q[:, :, :Lb])
        ks.append(k[:, :, :Sb])
        vs.append(v[:, :, :Sb])
    (qp, cq), (kp, ck), (vp, _) = _pack(qs), _pack(ks), _pack(vs)
    return qp, kp, vp, cq, ck, (qs, ks, vs)


VARLEN_LENGTHS = [(5, 5), (0, 3), (17, 40), (1, 1), (33, 33), (9, 100)]


def pin_varlen_equals_per_sequence_dense(varlen_attn):
    Hq, Hkv, D = 4, 2, 16
    qp, kp, vp, cq, ck, (qs, ks, vs) = _varlen_case(VARLEN_LENGTHS, Hq, Hkv, D, seed=50,
                                                     k_scale=2.0)
    for causal, window in [(True, 0), (True, 7), (False, 0)]:
        got = varlen_attn(qp, kp, vp, cq, ck, scale=0.4, causal=causal, window=window)
        for b, (Lb, Sb) in enumerate(VARLEN_LENGTHS):
            if Lb == 0:
                continue
            ref = oracle.attention(qs[b].contiguous(), ks[b].contiguous(), vs[b].contiguous(),
                                   scale=0.4, causal=causal, window=window)
            assert np.array_equal(got[cq[b]:cq[b + 1]], ref[0].transpose(1, 0, 2)), (b, causal)


def pin_varlen_equal_length_causal_rule(varlen_attn):
    """brotensor: key k of sequence b attends query q iff
    (k - cu_seqlens_k[b]) <= (q - cu_seqlens_q[b]).  With q = 0 every visible key
    gets the same weight; one-hot values make the visible set readable."""
    lengths = [(4, 4), (6, 6), (3, 3)]
    D = 8
    T = sum(L for L, _ in lengths)
    q = torch.zeros(T, 1, D).bfloat16()
    v = torch.zeros(T, 1, D)
    cu = np.concatenate([[0], np.cumsum([L for L, _ in lengths])]).astype(np.int32)
    for b, (L, _) in enumerate(lengths):
        for j in range(L):
            v[cu[b] + j, 0, j] = 1.0
    k = torch.randn(T, 1, D, generator=torch.Generator().manual_seed(3)).bfloat16()
    o = varlen_attn(q, k, v.bfloat16(), cu, cu, scale=1.0, causal=True)
    for b, (L, _) in enumerate(lengths):
        for i in range(L):
            expect = np.zeros(D)
            expect[:i + 1] = 1.0 / (i + 1)
            assert np.allclose(o[cu[b] + i, 0], expect, atol=1e-12), (b, i)


def pin_varlen_sequences_do_not_interact(varlen_attn):
    Hq, Hkv, D = 4, 2, 16
    qp, kp, vp, cq, ck, _ = _varlen_case(VARLEN_LENGTHS, Hq, Hkv, D, seed=60)
    base = varlen_attn(qp, kp, vp, cq, ck, scale=0.4, causal=True)
    kp2, vp2 = kp.clone(), vp.clone()
    kp2[ck[2]:ck[3]] = (-kp2[ck[2]:ck[3]].float() * 3).bfloat16()  # sequence 2's keys only
    vp2[ck[2]:ck[3]] = 5.0
    got = varlen_attn(qp, kp2, vp2, cq, ck, scale=0.4, causal=True)
    other = np.ones(qp.shape[0], dtype=bool)
    other[cq[2]:cq[3]] = False
    assert np.array_equal(got[other], base[other])
    assert not np.allclose(got[~other], base[~other])


VARLEN_PINS = [pin_varlen_equals_per_sequence_dense, pin_varlen_equal_length_causal_rule,
               pin_varlen_sequences_do_not_interact]


@pytest.mark.parametrize("pin", VARLEN_PINS, ids=lambda p: p.__name__)
def test_varlen_pin(pin):
    pin(oracle.attention_varlen)


@pytest.mark.parametrize("mutation", sorted(oracle.VARLEN_MUTATIONS))
def test_varlen_planted_mistake_fails_a_pin(mutation):
    def mutant(*a, **kw):
        return oracle.attention_varlen(*a, mutation=mutation, **kw)
    caught = []
    for pin in VARLEN_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutation {mutation} passed every pin"


def test_varlen_with_sinks_and_softcap_equals_per_sequence_dense():
    Hq, Hkv, D = 4, 2, 16
    lengths = [(7, 20), (12, 12), (1, 30)]
    qp, kp, vp, cq, ck, (qs, ks, vs) = _varlen_case(lengths, Hq, Hkv, D, seed=70, k_scale=3.0)
    sinks = torch.tensor([0.5, -1.0, 2.0, 0.0])
    got = oracle.attention_varlen(qp, kp, vp, cq, ck, scale=0.4, causal=True, window=9,
                                  softcap=2.5, sinks=sinks)
    for b in range(len(lengths)):
        ref = oracle.attention(qs[b].contiguous(), ks[b].contiguous(), vs[b].contiguous(),
                               scale=0.4, causal=True, window=9, softcap=2.5, sinks=sinks)
        assert np.array_equal(got[cq[b]:cq[b + 1]], ref[0].transpose(1, 0, 2))


def test_varlen_rejects_causal_sequences_shorter_in_keys():
    q = torch.zeros(5, 2, 8).bfloat16()
    k = torch.zeros(3, 2, 8).bfloat16()
    with pytest.raises(ValueError):
        oracle.attention_varlen(q, k, k, [0, 5], [0, 3], scale=1.0, causal=True)
    oracle.attention_varlen(q, k, k, [0, 5], [0, 3], scale=1.0, causal=False)
