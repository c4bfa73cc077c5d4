"""GPU parity of the two addressing modes against the fp64 oracle:
tfa_prefill_ring (rotating K/V cache, TensorFold's WINDOW/RING sliding layer)
and tfa_prefill_varlen (packed variable-length batches, brotensor's
flash_attention_varlen_forward), at the operator tolerance atol = rtol = 0.02
on the bf16 output."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, make_sinks, shaped, varlen_cu

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


def _assert_close(got, ref, what):
    got = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements off, max abs err {err.max():.4g}"


def _ring_from_dense(k_full, R, seed):
    """[B,H,R,D] ring holding positions [S-R, S) of k_full at row j mod R; the
    other rows hold large junk that must never be read as a visible key."""
    B, H, S, D = k_full.shape
    g = torch.Generator().manual_seed(seed)
    ring = (30.0 * torch.randn(B, H, R, D, generator=g)).bfloat16()
    lo = max(0, S - R)
    idx = torch.arange(lo, S)
    ring[:, :, idx % R] = k_full[:, :, lo:S]
    return ring


RING_CASES = [  # name, (B, Hq, Hkv, L, S, R, W, D), extras
    ("tensorfold_sliding_64x10000", (1, 8, 2, 64, 10000, 1088, 1024, 128), {}),
    ("chunk_300x4000", (2, 4, 2, 300, 4000, 1344, 1024, 128), {}),
    ("d64_200x700", (1, 4, 1, 200, 700, 512, 300, 64), {}),
    ("not_yet_wrapped", (1, 4, 2, 100, 300, 1024, 500, 128), {}),
    ("decode_l1", (2, 14, 2, 1, 9999, 1024, 1000, 128), {}),
    ("decode_l5_r576", (1, 8, 8, 5, 3000, 576, 500, 128), {}),
    ("softcap_sinks", (1, 8, 2, 130, 2500, 1152, 1000, 128), dict(softcap=20.0, sink_scale=2.0)),
]


@pytest.mark.parametrize("name,shape,extra", RING_CASES, ids=[c[0] for c in RING_CASES])
def test_ring_parity(name, shape, extra):
    B, Hq, Hkv, L, S, R, W, D = shape
    w = shaped(B, Hq, Hkv, L, S, D, k_scale=2.0, **extra)
    q, k, v, _ = make_inputs(w, seed=81)
    sinks = make_sinks(w, seed=81)
    kr, vr = _ring_from_dense(k, R, 1), _ring_from_dense(v, R, 2)
    o = tb.prefill_ring(q.cuda(), kr.cuda(), vr.cuda(), S=S, window=W, scale=w.softmax_scale,
                        softcap=w.softcap, sinks=sinks.cuda() if sinks is not None else None)
    tb.check_status()
    ref = oracle.attention_ring(q, kr, vr, S=S, scale=w.softmax_scale, window=W,
                                softcap=w.softcap, sinks=sinks)
    _assert_close(o, ref, name)


def test_ring_rejections():
    q = torch.zeros(1, 4, 10, 128, dtype=torch.bfloat16, device="cuda")
    kr = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16, device="cuda")
    for kw, code in [(dict(S=100, window=0), tb.TFA_ERR_RING),    # a ring needs a window
                     (dict(S=100, window=60), tb.TFA_ERR_RING),   # 64 < 60 - 1 + 10
                     (dict(S=5, window=8), tb.TFA_ERR_SHAPE)]:    # S < L
        with pytest.raises(tb.TfaError) as e:
            tb.prefill_ring(q, kr, kr, **kw)
        assert e.value.code == code
    kr96 = torch.zeros(1, 2, 96, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tb.TfaError) as e:
        tb.prefill_ring(q, kr96, kr96, S=100, window=8)  # not a multiple of 64
    assert e.value.code == tb.TFA_ERR_RING


def _varlen_inputs(lengths, Hq, Hkv, D, seed, k_scale=1.0):
    qs, ks, vs = [], [], []
    for n, (Lb, Sb) in enumerate(lengths):
        q, k, v, _ = make_inputs(shaped(1, Hq, Hkv, max(Lb, 1), max(Sb, 1), D, k_scale=k_scale),
                                 seed=seed + n)
        qs.append(q[0, :, :Lb].transpose(0, 1))
        ks.append(k[0, :, :Sb].transpose(0, 1))
        vs.append(v[0, :, :Sb].transpose(0, 1))
    cq = np.concatenate([[0], np.cumsum([L for L, _ in lengths])]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum([S for _, S in lengths])]).astype(np.int32)
    return (torch.cat(qs).contiguous(), torch.cat(ks).contiguous(), torch.cat(vs).contiguous(),
            cq, ck)


VARLEN_CASES = [  # name, lengths, (Hq, Hkv, D), causal, window, extras
    ("mixed_causal", [(300, 300), (1, 1), (0, 5), (129, 700), (1000, 1000), (7, 7)],
     (8, 2, 128), True, 0, {}),
    ("mixed_bidirectional", [(50, 400), (256, 256), (3, 1000), (131, 9)], (4, 4, 128), False, 0, {}),
    ("window", [(500, 900), (260, 260), (10, 2000)], (8, 2, 128), True, 129, {}),
    ("d64_gqa", [(200, 300), (513, 513), (1, 64)], (12, 4, 64), True, 0, {}),
    ("many_short", [(int(n), int(n) + int(m)) for n, m in
                    zip(np.random.default_rng(3).integers(1, 90, 64),
                        np.random.default_rng(4).integers(0, 300, 64))], (4, 2, 128), True, 0, {}),
    ("softcap_sinks", [(128, 128), (300, 800), (5, 5)], (8, 2, 128), True, 0,
     dict(softcap=10.0, sinks=True)),
    # the most sequences a call takes: the device-side sort of the compact
    # item deal runs over all 1024 (lengths 0..299, ties and empty sequences)
    ("max_seqs", [(int(n), int(n)) for n in np.random.default_rng(5).integers(0, 300, 1024)],
     (2, 1, 64), True, 0, {}),
    # a bound beyond the compact deal's group table: the plain item grid
    ("bound_past_compact_deal", [(300, 300), (1, 40), (700, 900)], (4, 2, 128), True, 0,
     dict(max_seqlen_q=1024 * 256 + 1)),
]


@pytest.mark.parametrize("name,lengths,heads,causal,window,extra", VARLEN_CASES,
                         ids=[c[0] for c in VARLEN_CASES])
def test_varlen_parity(name, lengths, heads, causal, window, extra):
    Hq, Hkv, D = heads
    q, k, v, cq, ck = _varlen_inputs(lengths, Hq, Hkv, D, seed=90, k_scale=2.0)
    softcap = extra.get("softcap", 0.0)
    sinks = torch.linspace(-2.0, 2.0, Hq) if extra.get("sinks") else None
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    o = tb.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cq).cuda(),
                          torch.from_numpy(ck).cuda(),
                          max_seqlen_q=extra.get("max_seqlen_q", max(L for L, _ in lengths)),
                          scale=1 / np.sqrt(D), causal=causal, window=window, softcap=softcap,
                          sinks=sinks.cuda() if sinks is not None else None, out=out)
    tb.check_status()
    ref = oracle.attention_varlen(q, k, v, cq, ck, scale=1 / np.sqrt(D), causal=causal,
                                  window=window, softcap=softcap, sinks=sinks)
    _assert_close(o, ref, name)


def test_varlen_bad_seqlens_are_reported_and_skipped():
    lengths = [(100, 100), (50, 80), (30, 300)]
    Hq, Hkv, D = 4, 2, 128
    q, k, v, cq, ck = _varlen_inputs(lengths, Hq, Hkv, D, seed=95)
    bad_k = ck.copy()
    bad_k[2] = bad_k[1] + 10  # sequence 1: 10 keys for 50 causal queries
    out = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
    tb.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cq).cuda(),
                      torch.from_numpy(bad_k).cuda(), max_seqlen_q=100, causal=True, out=out)
    with pytest.raises(tb.TfaError) as e:
        tb.check_status()
    assert e.value.code == tb.TFA_ERR_SEQLENS
    assert torch.all(out[cq[1]:cq[2]] == 0)  # the bad sequence was not written
    tb.check_status()  # the report was cleared
    # a sequence longer than max_seqlen_q is reported too
    tb.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cq).cuda(),
                      torch.from_numpy(ck).cuda(), max_seqlen_q=60, causal=True, out=out)
    with pytest.raises(tb.TfaError) as e:
        tb.check_status()
    assert e.value.code == tb.TFA_ERR_SEQLENS


def test_varlen_empty_and_rejected_calls():
    q = torch.zeros(0, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(5, 2, 128, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    tb.prefill_varlen(q, k, k, cu, torch.tensor([0, 5], dtype=torch.int32, device="cuda"),
                      max_seqlen_q=0)  # no query row: nothing to do
    q1 = torch.zeros(3, 4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tb.TfaError) as e:  # window without causal
        tb.prefill_varlen(q1, k, k, torch.tensor([0, 3], dtype=torch.int32, device="cuda"),
                          torch.tensor([0, 5], dtype=torch.int32, device="cuda"), max_seqlen_q=3,
                          causal=False, window=4)
    assert e.value.code == tb.TFA_ERR_WINDOW


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if w.kind in ("ring", "varlen")])
def test_full_size_workloads_sampled(name):
    """The benchmark's rotating-cache and variable-length workloads, launched as
    the benchmark launches them, on rows the oracle computes one by one."""
    w = WORKLOADS[name]
    q, k, v, _ = make_inputs(w, seed=0)
    sinks = make_sinks(w, seed=0)
    rng = np.random.default_rng(5)
    if w.kind == "ring":
        o = tb.prefill_ring(q.cuda(), k.cuda(), v.cuda(), S=w.S, window=w.window,
                            scale=w.softmax_scale, softcap=w.softcap,
                            sinks=sinks.cuda() if sinks is not None else None)
        tb.check_status()
        n = w.B * w.Hq * w.L
        rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(n, 600), replace=False)]))
        ref = oracle.attention_ring(q, k, v, S=w.S, scale=w.softmax_scale, window=w.window,
                                    softcap=w.softcap, sinks=sinks, rows=rows)
        got = o.reshape(-1, w.D)[torch.as_tensor(rows, device=o.device)]
        _assert_close(got, ref, name)
        return
    cq, ck = varlen_cu(w)
    o = tb.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cq).cuda(),
                          torch.from_numpy(ck).cuda(), max_seqlen_q=w.L, scale=w.softmax_scale,
                          causal=w.causal, window=w.window, softcap=w.softcap,
                          sinks=sinks.cuda() if sinks is not None else None)
    tb.check_status()
    for b in [0, 4, 8, 12, len(w.seqlens) - 1]:  # sampled rows of several sequences
        L, S = w.seqlens[b]
        qb = q[cq[b]:cq[b + 1]].transpose(0, 1)[None].contiguous()
        kb = k[ck[b]:ck[b + 1]].transpose(0, 1)[None].contiguous()
        vb = v[ck[b]:ck[b + 1]].transpose(0, 1)[None].contiguous()
        i = np.unique(np.concatenate([[0, 127, 128, L - 1], rng.choice(L, size=min(L, 24), replace=False)]))
        i = i[i < L]
        rows = (np.arange(w.Hq)[:, None] * L + i[None, :]).reshape(-1)
        ref = oracle.attention(qb, kb, vb, scale=w.softmax_scale, causal=w.causal, window=w.window,
                               softcap=w.softcap, sinks=sinks, rows=rows)
        got = o[cq[b]:cq[b + 1]].transpose(0, 1).reshape(-1, w.D)[torch.as_tensor(rows, device=o.device)]
        _assert_close(got, ref, f"{name} sequence {b}")
