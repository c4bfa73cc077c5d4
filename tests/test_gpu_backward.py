"""GPU parity of the backward pass (tfa_prefill_backward) against the fp64
oracle's gradients on the same seeded inputs.

Bar, from the arithmetic.  Each gradient element is a sum of products whose
one non-exact factor was rounded to bf16 (relative error <= 2^-9): P^T in
dV = P^T dO, dS in dQ = scale dS K and dK = scale dS^T Q; dS also inherits
the rounding of the recomputed output O (bf16) through
delta = rowsum(dO o O); the result is rounded to bf16 (2^-9 relative).  So,
per element, with A the sum of the absolute values of its terms:
    |gpu - ref| <= 2^-8 A + 2^-8 |ref| + 2^-8 scale E_delta
twice the one-rounding bound, where E_delta is the delta term
sum_j P |dO||O| |K| (dQ) or sum_i P |dO||O| |Q| (dK).  A is computed from the
oracle's softmax weights and plain products of the inputs; the values
compared against are the oracle's gradients."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_dout, make_inputs, shaped

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -8


def _dout(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed)).bfloat16()


def _bounds(w, q, k, v, do, km):
    """Per-element error bounds (dq, dk, dv) of the derivation above."""
    Q, K, V, dO = (t.double().numpy() for t in (q, k, v, do))
    O = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window, key_mask=km)
    G = w.Hq // w.Hkv
    bq = np.zeros(Q.shape)
    bk = np.zeros(K.shape)
    bv = np.zeros(V.shape)
    s = w.softmax_scale
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // G
            P = oracle.softmax_weights(q, k, b=b, h=h, scale=s, causal=w.causal, window=w.window,
                                       key_mask=km)
            dP = dO[b, h] @ V[b, g].T
            delta = (P * dP).sum(1, keepdims=True)
            dS = np.abs(P * (dP - delta))
            e_delta = np.abs(dO[b, h] * O[b, h]).sum(1, keepdims=True)  # per row
            bq[b, h] += EPS * s * (dS @ np.abs(K[b, g]) + (P * e_delta) @ np.abs(K[b, g]))
            bk[b, g] += EPS * s * (dS.T @ np.abs(Q[b, h]) + (P * e_delta).T @ np.abs(Q[b, h]))
            bv[b, g] += EPS * (P.T @ np.abs(dO[b, h]))
    return bq, bk, bv


def _check(got, ref, bound, what):
    got = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    err = np.abs(got - ref)
    lim = bound + EPS * np.abs(ref) + 1e-6
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements off, worst ratio "
                           f"{(err / lim).max():.3g}")
    return float((err / lim).max())


CASES = [
    ("witness_33x47", shaped(1, 8, 2, 33, 47, 128)),
    ("causal_130x300", shaped(2, 4, 2, 130, 300, 128)),
    ("no_prefix_257", shaped(1, 4, 4, 257, 257, 128)),
    ("group7_200x450", shaped(1, 14, 2, 200, 450, 128)),
    ("window129", shaped(1, 4, 2, 300, 700, 128, window=129)),
    ("keymask", shaped(2, 4, 2, 200, 450, 128, key_mask_keep=0.6)),
    ("bidirectional", shaped(1, 4, 2, 190, 333, 128, causal=False, k_scale=3.0)),
    ("d64", shaped(1, 6, 3, 300, 600, 64)),
    ("d64_window_mask", shaped(1, 4, 2, 260, 900, 64, window=300, key_mask_keep=0.8)),
    ("decode_l1", shaped(2, 14, 2, 1, 1000, 128)),
    ("decode_l5_window", shaped(1, 8, 2, 5, 700, 128, window=200)),
    ("long_keys_split", shaped(1, 2, 1, 256, 20000, 128, k_scale=2.0)),
    # more items than CTAs, each with 1-4 key tiles: a CTA moves to its next
    # item while the tensor core may have run two score tiles ahead
    ("multi_item_short_ranges", shaped(2, 32, 4, 512, 512, 128)),
]


@pytest.mark.parametrize("name,w", CASES, ids=[n for n, _ in CASES])
def test_backward_parity(name, w):
    q, k, v, km = make_inputs(w, seed=61)
    do = _dout(q.shape, 62)
    dq, dk, dv = tb.backward(q.cuda(), k.cuda(), v.cuda(), do.cuda(), scale=w.softmax_scale,
                             causal=w.causal, window=w.window,
                             key_mask=km.cuda() if km is not None else None)
    tb.check_status()
    rq, rk, rv = oracle.attention_backward(q, k, v, do, scale=w.softmax_scale, causal=w.causal,
                                           window=w.window, key_mask=km)
    bq, bk, bv = _bounds(w, q, k, v, do, km)
    errs = [_check(dq, rq, bq, f"{name} dq"), _check(dk, rk, bk, f"{name} dk"),
            _check(dv, rv, bv, f"{name} dv")]
    print(name, "worst error / bound", [f"{e:.3g}" for e in errs])


def test_backward_fully_masked_batch_is_zero():
    w = shaped(2, 4, 2, 150, 300, 128, key_mask_keep=0.7)
    q, k, v, km = make_inputs(w, seed=63)
    km[1] = 0.0
    do = _dout(q.shape, 64)
    dq, dk, dv = tb.backward(q.cuda(), k.cuda(), v.cuda(), do.cuda(), causal=True, key_mask=km.cuda())
    tb.check_status()
    assert torch.all(dq[1] == 0) and torch.all(dk[1] == 0) and torch.all(dv[1] == 0)


def test_backward_keys_no_row_sees_are_zero():
    # window 64 and prefix 1000: keys before position ~936 are seen by no row
    w = shaped(1, 4, 2, 100, 1100, 128, window=64)
    q, k, v, _ = make_inputs(w, seed=65)
    do = _dout(q.shape, 66)
    dq, dk, dv = tb.backward(q.cuda(), k.cuda(), v.cuda(), do.cuda(), causal=True, window=64)
    tb.check_status()
    assert torch.all(dk[:, :, :900] == 0) and torch.all(dv[:, :, :900] == 0)
    rq, rk, rv = oracle.attention_backward(q, k, v, do, scale=w.softmax_scale, causal=True, window=64)
    bq, bk, bv = _bounds(w, q, k, v, do, None)
    _check(dq, rq, bq, "dq")
    _check(dk, rk, bk, "dk")
    _check(dv, rv, bv, "dv")


def _row_softmax(scores, allowed):
    s = np.where(allowed, scores, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(allowed, np.exp(s - m), 0.0)
    d = e.sum(axis=-1, keepdims=True)
    return e / np.where(d > 0, d, 1.0)


def test_backward_full_size_sampled():
    """The benchmark's backward workload, launched as the benchmark launches it:
    dQ on sampled rows and dK/dV on sampled keys of one KV group against the
    oracle's row entries, with the per-element bound of the small cases."""
    w = WORKLOADS["llama_gqa_chunk_2048x8192_backward"]
    q, k, v, km = make_inputs(w, seed=0)
    do = make_dout(w, seed=0)
    dq, dk, dv = tb.backward(q.cuda(), k.cuda(), v.cuda(), do.cuda(), scale=w.softmax_scale,
                             causal=w.causal, window=w.window)
    tb.check_status()
    s, G, P0 = w.softmax_scale, w.Hq // w.Hkv, w.S - w.L
    Q, K, V, dO = (t.double().numpy() for t in (q, k, v, do))
    keys_all = np.arange(w.S)
    # dQ rows
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, w.L - 1, 127, 128, 1023, 2047],
                                     rng.integers(0, w.Hq * w.L, 58)]))
    ref = oracle.attention_backward_dq_rows(q, k, v, do, rows, scale=s, causal=True)
    O = oracle.attention(q, k, v, scale=s, causal=True, rows=rows)
    got = dq.reshape(-1, w.D)[torch.as_tensor(rows, device=dq.device)]
    bound = np.zeros_like(ref)
    for n, row in enumerate(rows):
        h, i = divmod(int(row), w.L)
        g = h // G
        allowed = keys_all <= P0 + i
        Prow = _row_softmax(s * (K[0, g] @ Q[0, h, i]), allowed)
        dP = V[0, g] @ dO[0, h, i]
        dS = Prow * (dP - (Prow * dP).sum())
        e = np.abs(dO[0, h, i] * O[n]).sum()
        bound[n] = EPS * s * (np.abs(dS) @ np.abs(K[0, g]) + e * (Prow @ np.abs(K[0, g])))
    ratio = _check(got, ref, bound, "full-size dq rows")
    # dK / dV of sampled keys of the last KV group
    g = w.Hkv - 1
    keys = np.unique(np.concatenate([[0, 127, 128, 6143, 6144, 8191], rng.integers(0, w.S, 18)]))
    rk, rv = oracle.attention_backward_kv_rows(q, k, v, do, b=0, g=g, keys=keys, scale=s, causal=True)
    bk = np.zeros_like(rk)
    bv = np.zeros_like(rv)
    allowed = keys_all[None, :] <= P0 + np.arange(w.L)[:, None]
    for h in range(g * G, (g + 1) * G):
        Ph = _row_softmax(s * (Q[0, h] @ K[0, g].T), allowed)
        dPh = dO[0, h] @ V[0, g].T
        dSh = Ph * (dPh - (Ph * dPh).sum(axis=1, keepdims=True))
        Oh = Ph @ V[0, g]
        eh = np.abs(dO[0, h] * Oh).sum(axis=1)
        bv += EPS * (Ph[:, keys].T @ np.abs(dO[0, h]))
        bk += EPS * s * (np.abs(dSh[:, keys]).T @ np.abs(Q[0, h]) + (Ph[:, keys] * eh[:, None]).T @ np.abs(Q[0, h]))
    kk = torch.as_tensor(keys, device=dk.device)
    rk_ratio = _check(dk[0, g][kk], rk, bk, "full-size dk rows")
    rv_ratio = _check(dv[0, g][kk], rv, bv, "full-size dv rows")
    print("full size worst error / bound", f"{ratio:.3g} {rk_ratio:.3g} {rv_ratio:.3g}")


SAVED_CASES = [
    ("causal_130x300", shaped(2, 4, 2, 130, 300, 128)),
    ("d64_window_mask", shaped(1, 6, 3, 260, 900, 64, window=300, key_mask_keep=0.8)),
    ("decode_l1", shaped(2, 14, 2, 1, 1000, 128)),
    ("bidirectional", shaped(1, 4, 2, 190, 333, 128, causal=False, k_scale=3.0)),
    ("fully_masked_batch", shaped(2, 4, 2, 150, 300, 128, key_mask_keep=0.7)),
]


def _saved_inputs(name, w):
    q, k, v, km = make_inputs(w, seed=71)
    if name == "fully_masked_batch":
        km[1] = 0.0
    do = _dout(q.shape, 72)
    return q, k, v, km, do


@pytest.mark.parametrize("name,w", SAVED_CASES, ids=[n for n, _ in SAVED_CASES])
def test_saved_backward_is_the_recompute_backward(name, w):
    """tfa_prefill_backward_saved on tfa_prefill_lse's (o, lse) gives the
    recompute-based backward's gradients bit for bit (same kernels, same
    statistics)."""
    q, k, v, km, do = _saved_inputs(name, w)
    Q, K, V, DO = (t.cuda() for t in (q, k, v, do))
    KM = km.cuda() if km is not None else None
    kw = dict(scale=w.softmax_scale, causal=w.causal, window=w.window, key_mask=KM)
    o, lse = tb.prefill_lse(Q, K, V, **kw)
    saved = tb.backward(Q, K, V, DO, saved=(o, lse), **kw)
    recomputed = tb.backward(Q, K, V, DO, **kw)
    tb.check_status()
    for a, b, n in zip(saved, recomputed, ("dq", "dk", "dv")):
        assert torch.equal(a, b), f"{name}: {n} differs"


@pytest.mark.parametrize("name,w", SAVED_CASES, ids=[n for n, _ in SAVED_CASES])
def test_lse_is_the_log_sum_exp(name, w):
    """lse[b,h,i] = log2 sum_j exp(scale q.k_j) over the allowed keys, +inf for
    a row with none.  Bound: the fp32 score sum (D products of bf16 values)
    errs by at most D 2^-24 sum|q k| per score, and exp2.approx by ~2^-22
    relative; both stay far below the 1e-3 (log2 units) asserted here.  The
    output is checked against the oracle at the usual 0.02."""
    q, k, v, km, _ = _saved_inputs(name, w)
    Q, K, V = (t.cuda() for t in (q, k, v))
    KM = km.cuda() if km is not None else None
    o, lse = tb.prefill_lse(Q, K, V, scale=w.softmax_scale, causal=w.causal, window=w.window,
                            key_mask=KM)
    tb.check_status()
    ref_o = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                             key_mask=km)
    got_o = o.float().cpu().double().numpy()
    assert np.allclose(got_o, ref_o, atol=0.02, rtol=0.02)
    G = w.Hq // w.Hkv
    P0 = w.S - w.L
    i = np.arange(w.L)[:, None]
    j = np.arange(w.S)[None, :]
    allowed = np.ones((w.L, w.S), dtype=bool)
    if w.causal:
        allowed &= j <= P0 + i
        if w.window > 0:
            allowed &= j > P0 + i - w.window
    got = lse.cpu().double().numpy()
    Qd, Kd = q.double().numpy(), k.double().numpy()
    for b in range(w.B):
        al = allowed if km is None else allowed & (km[b].numpy() > 0.5)[None, :]
        for h in range(w.Hq):
            s = w.softmax_scale * (Qd[b, h] @ Kd[b, h // G].T)
            s = np.where(al, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            empty = ~al.any(axis=1)
            mm = np.where(np.isfinite(m), m, 0.0)
            ref = (mm[:, 0] + np.log(np.exp(s - mm).sum(axis=1))) / np.log(2.0)
            g = got[b, h]
            assert np.all(np.isposinf(g[empty])), f"{name}: empty rows must be +inf"
            assert np.all(np.abs(g[~empty] - ref[~empty]) <= 1e-3), \
                f"{name}: worst {np.abs(g[~empty] - ref[~empty]).max():.3g}"
