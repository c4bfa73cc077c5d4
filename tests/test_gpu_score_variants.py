"""GPU parity of the score variants (tfa_attention_ex): the logit softcap of
brotensor flash_attention.h's Gemma-2 extensions and per-head attention sinks,
against the fp64 oracle on the same seeded inputs, at the operator tolerance
(atol = rtol = 0.02 on the bf16 output).  Cases cover the prefill and the
short-query (packed) paths, both schedules (whole query tiles and key ranges
split across CTAs, whose merge must carry the sink exactly once), the key
mask, windows, bidirectional attention and D = 64."""
import math

import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import make_inputs, make_sinks, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


def _assert_close(got, ref, what):
    got = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements off, max abs err {err.max():.4g}"


def _run(w, seed, sinks=None):
    q, k, v, km = make_inputs(w, seed)
    if sinks is None:
        sinks = make_sinks(w, seed)
    o = tb.prefill(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=w.causal,
                   window=w.window, key_mask=km.cuda() if km is not None else None,
                   softcap=w.softcap, sinks=sinks.cuda() if sinks is not None else None)
    tb.check_status()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km, softcap=w.softcap, sinks=sinks)
    return o, ref, (q, k, v, km, sinks)


CASES = [
    # prefill path
    ("softcap50_witness", shaped(1, 8, 2, 33, 47, 128, softcap=50.0, k_scale=4.0)),
    ("softcap5_ragged", shaped(2, 4, 2, 130, 300, 128, softcap=5.0, k_scale=4.0)),
    ("softcap1_window", shaped(1, 4, 2, 300, 700, 128, window=129, softcap=1.0, k_scale=4.0)),
    ("softcap_keymask", shaped(2, 4, 2, 200, 450, 128, key_mask_keep=0.5, softcap=8.0, k_scale=4.0)),
    ("softcap_bidirectional", shaped(1, 4, 2, 257, 500, 128, causal=False, softcap=3.0, k_scale=4.0)),
    ("softcap_d64", shaped(1, 4, 2, 300, 600, 64, softcap=4.0, k_scale=4.0)),
    ("sinks_witness", shaped(1, 8, 2, 33, 47, 128, sink_scale=2.0)),
    ("sinks_window1", shaped(1, 4, 2, 140, 400, 128, window=1, sink_scale=1.0)),
    ("sinks_keymask_sparse", shaped(2, 4, 2, 150, 600, 128, key_mask_keep=0.05, sink_scale=3.0)),
    ("sinks_softcap_d64_bidir", shaped(1, 6, 3, 200, 333, 64, causal=False, softcap=6.0,
                                       sink_scale=2.0, k_scale=4.0)),
    # key ranges cut across CTAs (few items, long keys): the merge adds the sink once
    ("split_sinks_softcap", shaped(1, 2, 1, 300, 40000, 128, softcap=20.0, sink_scale=2.0,
                                   k_scale=4.0)),
    ("split_sinks_keymask_d64", shaped(1, 2, 1, 256, 30000, 64, key_mask_keep=0.9, sink_scale=1.0)),
    # short queries (packed tiles; long keys are split across CTAs)
    ("decode_l1_softcap_sinks", shaped(1, 56, 8, 1, 8192, 128, softcap=30.0, sink_scale=2.0,
                                       k_scale=4.0)),
    ("decode_l3_window_keymask_sinks", shaped(2, 8, 2, 3, 3000, 128, window=700, key_mask_keep=0.7,
                                              softcap=10.0, sink_scale=1.0)),
    ("decode_l8_d64_sinks", shaped(1, 32, 2, 8, 2000, 64, sink_scale=2.0)),
    ("decode_l1_long_split", shaped(1, 8, 8, 1, 65536, 128, softcap=15.0, sink_scale=2.0,
                                    k_scale=4.0)),
]


@pytest.mark.parametrize("name,w", CASES, ids=[n for n, _ in CASES])
def test_score_variant_parity(name, w):
    o, ref, _ = _run(w, seed=41)
    _assert_close(o, ref, name)


@pytest.mark.parametrize("L", [1, 5, 100])
def test_sinks_on_fully_masked_rows_give_zeros(L):
    w = shaped(2, 4, 2, L, 300, 128, key_mask_keep=0.5, sink_scale=2.0)
    q, k, v, km = make_inputs(w, 3)
    km[1] = 0.0  # every row of batch 1 sees no key
    sinks = make_sinks(w, 3).cuda()
    o = tb.prefill(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=True,
                   key_mask=km.cuda(), sinks=sinks)
    tb.check_status()
    assert torch.all(o[1] == 0)
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, key_mask=km,
                           sinks=sinks.cpu())
    _assert_close(o, ref, "fully masked with sinks")


@pytest.mark.parametrize("L", [1, 300])
def test_dominant_sink_drives_output_to_zero(L):
    w = shaped(1, 4, 2, L, 2000, 128)
    sinks = torch.full((4,), 200.0)  # e^(200 - m) dwarfs every score's weight
    o, ref, _ = _run(w, seed=5, sinks=sinks)
    assert float(o.abs().max()) < 1e-30
    assert np.abs(ref).max() < 1e-30


@pytest.mark.parametrize("L", [1, 7, 300])
def test_minus_infinite_sinks_are_bit_identical_to_no_sinks(L):
    w = shaped(1, 8, 2, L, 3000, 128, key_mask_keep=0.8)
    q, k, v, km = make_inputs(w, 6)
    dq, dk, dv, dkm = q.cuda(), k.cuda(), v.cuda(), km.cuda()
    plain = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, key_mask=dkm)
    neg = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, key_mask=dkm,
                     sinks=torch.full((8,), -math.inf, device="cuda"))
    tb.check_status()
    assert torch.equal(plain, neg)


def test_huge_softcap_matches_the_uncapped_oracle():
    w = shaped(1, 4, 2, 200, 900, 128, k_scale=4.0, softcap=1e6)
    o, _, (q, k, v, km, _) = _run(w, seed=8)
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True)
    _assert_close(o, ref, "softcap 1e6 vs no cap")


@pytest.mark.parametrize("over,code", [
    (dict(softcap=-1.0), tb.TFA_ERR_SOFTCAP),
    (dict(softcap=float("nan")), tb.TFA_ERR_SOFTCAP),
])
def test_bad_softcap_is_rejected(over, code):
    q = torch.zeros(1, 4, 33, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 47, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tb.TfaError) as e:
        tb.prefill(q, k, k, causal=True, **over)
    assert e.value.code == code
