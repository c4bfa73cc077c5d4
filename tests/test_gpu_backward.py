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
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped

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
