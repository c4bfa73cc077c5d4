"""Pins for the oracle's backward (gradients of the plain definition), each
independent of the backward code: torch's own autograd through its scaled
dot-product attention in float64, central finite differences of the forward
oracle, exact zeros for excluded keys, and the GQA sum over a group.  Planted
mistakes must fail at least one pin."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped


def _dout(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed)).bfloat16()


def _allowed(L, S, causal, window, km, B):
    P = S - L
    a = torch.ones(L, S, dtype=torch.bool)
    if causal:
        a = a.tril(diagonal=P)
        if window > 0:
            a &= ~torch.ones(L, S, dtype=torch.bool).tril(diagonal=P - window)
    a = a[None, None].expand(B, 1, L, S)
    if km is not None:
        a = a & (km > 0.5)[:, None, None, :]
    return a


def pin_matches_torch_autograd(bwd):
    """torch.nn.functional.scaled_dot_product_attention in float64 with GQA and a
    boolean mask, differentiated by autograd (rows keep >= 1 allowed key)."""
    for (B, Hq, Hkv, L, S, D, causal, window, keep, scale) in [
            (1, 4, 2, 9, 23, 16, True, 0, None, 0.3),
            (2, 6, 3, 12, 12, 32, True, 5, None, 0.25),
            (1, 4, 4, 7, 19, 16, False, 0, 0.7, 0.4),
            (2, 8, 2, 5, 30, 16, True, 0, 0.8, 0.35)]:
        q, k, v, km = make_inputs(shaped(B, Hq, Hkv, L, S, D, key_mask_keep=keep, k_scale=2.0),
                                  seed=L + S)
        if km is not None:
            km[:, -1] = 1.0  # the last key is visible to every causal row: no empty row
        do = _dout(q.shape, 7)
        qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
        allowed = _allowed(L, S, causal, window, km, B)
        out = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=allowed, scale=scale,
                                             enable_gqa=True)
        out.backward(do.double())
        dq, dk, dv = bwd(q, k, v, do, scale=scale, causal=causal, window=window, key_mask=km)
        for got, ref in [(dq, qd.grad), (dk, kd.grad), (dv, vd.grad)]:
            assert np.allclose(got, ref.numpy(), atol=1e-11, rtol=1e-9)


def pin_finite_differences_of_the_forward(bwd):
    """d/dx of sum(dout * O) by central differences of the forward oracle, at
    entries whose +/- step is exact in bf16 (x = +-1, step 2^-7)."""
    B, Hq, Hkv, L, S, D, scale = 1, 4, 2, 6, 11, 16, 0.2
    q, k, v, _ = make_inputs(shaped(B, Hq, Hkv, L, S, D), seed=21)
    do = _dout(q.shape, 22)
    for causal, window in [(True, 0), (True, 4), (False, 0)]:
        dq, dk, dv = bwd(q, k, v, do, scale=scale, causal=causal, window=window)
        h = 2.0 ** -7

        def loss(qq, kk, vv):
            o = oracle.attention(qq, kk, vv, scale=scale, causal=causal, window=window)
            return float((o * do.double().numpy()).sum())

        for name, grad, idx in [("q", dq, (0, 1, 3, 5)), ("q", dq, (0, 3, 0, 2)),
                                ("k", dk, (0, 0, 4, 7)), ("k", dk, (0, 1, 10, 1)),
                                ("v", dv, (0, 1, 2, 9)), ("v", dv, (0, 0, 8, 0))]:
            plus = {"q": q.clone(), "k": k.clone(), "v": v.clone()}
            minus = {"q": q.clone(), "k": k.clone(), "v": v.clone()}
            plus[name][idx] = 1.0 + h
            minus[name][idx] = 1.0 - h
            base = {"q": q.clone(), "k": k.clone(), "v": v.clone()}
            base[name][idx] = 1.0
            # the gradient at x = 1 (the oracle's, recomputed there)
            g = bwd(base["q"], base["k"], base["v"], do, scale=scale, causal=causal, window=window)
            gx = {"q": g[0], "k": g[1], "v": g[2]}[name][idx]
            fd = (loss(plus["q"], plus["k"], plus["v"]) - loss(minus["q"], minus["k"], minus["v"])) / (2 * h)
            assert abs(fd - gx) <= 2e-4 * max(1.0, abs(gx)), (name, idx, causal, fd, gx)


def pin_excluded_keys_get_no_gradient(bwd):
    B, Hq, Hkv, L, S, D = 2, 4, 2, 8, 20, 16
    q, k, v, km = make_inputs(shaped(B, Hq, Hkv, L, S, D, key_mask_keep=0.6), seed=31)
    do = _dout(q.shape, 32)
    _, dk, dv = bwd(q, k, v, do, scale=0.3, causal=True, window=0, key_mask=km)
    dropped = (km <= 0.5).numpy()
    for b in range(B):
        assert np.all(dk[b][:, dropped[b]] == 0.0) and np.all(dv[b][:, dropped[b]] == 0.0)
    # keys beyond every row's causal reach (none here: P = S - L covers them) and a
    # fully masked batch: all gradients exactly zero
    km2 = km.clone()
    km2[1] = 0.0
    dq, dk, dv = bwd(q, k, v, do, scale=0.3, causal=True, window=0, key_mask=km2)
    assert np.all(dq[1] == 0.0) and np.all(dk[1] == 0.0) and np.all(dv[1] == 0.0)


def pin_gqa_gradient_is_the_group_sum(bwd):
    B, Hq, Hkv, L, S, D, G = 1, 6, 2, 7, 15, 16, 3
    q, k, v, _ = make_inputs(shaped(B, Hq, Hkv, L, S, D), seed=41)
    do = _dout(q.shape, 42)
    dq, dk, dv = bwd(q, k, v, do, scale=0.3, causal=True, window=3)
    dq_r, dk_r, dv_r = bwd(q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), do, scale=0.3,
                           causal=True, window=3)
    assert np.allclose(dq, dq_r, atol=1e-13, rtol=0)
    assert np.allclose(dk, dk_r.reshape(B, Hkv, G, S, D).sum(2), atol=1e-12, rtol=0)
    assert np.allclose(dv, dv_r.reshape(B, Hkv, G, S, D).sum(2), atol=1e-12, rtol=0)


BACKWARD_PINS = [pin_matches_torch_autograd, pin_finite_differences_of_the_forward,
                 pin_excluded_keys_get_no_gradient, pin_gqa_gradient_is_the_group_sum]


@pytest.mark.parametrize("pin", BACKWARD_PINS, ids=lambda p: p.__name__)
def test_backward_pin(pin):
    pin(oracle.attention_backward)


@pytest.mark.parametrize("mutation", sorted(oracle.BACKWARD_MUTATIONS))
def test_backward_planted_mistake_fails_a_pin(mutation):
    def mutant(*a, **kw):
        return oracle.attention_backward(*a, mutation=mutation, **kw)
    caught = []
    for pin in BACKWARD_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutation {mutation} passed every pin"


def test_dq_rows_equal_the_full_backward():
    """The per-row dQ entry (used at sizes the full oracle cannot reach) against
    the full oracle backward (itself pinned above)."""
    w = shaped(2, 6, 2, 40, 90, 32, key_mask_keep=0.8)
    q, k, v, km = make_inputs(w, seed=81)
    do = _dout(q.shape, 82)
    for causal, window in [(True, 0), (True, 9), (False, 0)]:
        dq, _, _ = oracle.attention_backward(q, k, v, do, scale=0.3, causal=causal, window=window,
                                             key_mask=km)
        rows = np.array([0, 5, 39, 40, 41, 150, 479], dtype=np.int64)
        got = oracle.attention_backward_dq_rows(q, k, v, do, rows, scale=0.3, causal=causal,
                                                window=window, key_mask=km)
        assert np.array_equal(got, dq.reshape(-1, w.D)[rows])


def test_kv_rows_equal_the_full_backward():
    w = shaped(2, 6, 2, 40, 90, 32, key_mask_keep=0.8)
    q, k, v, km = make_inputs(w, seed=83)
    do = _dout(q.shape, 84)
    for causal, window in [(True, 0), (True, 9), (False, 0)]:
        _, dk, dv = oracle.attention_backward(q, k, v, do, scale=0.3, causal=causal, window=window,
                                              key_mask=km)
        keys = [0, 3, 49, 50, 88, 89]
        for b, g in [(0, 0), (1, 1)]:
            gk, gv = oracle.attention_backward_kv_rows(q, k, v, do, b=b, g=g, keys=keys, scale=0.3,
                                                       causal=causal, window=window, key_mask=km)
            assert np.allclose(gk, dk[b, g, keys], atol=1e-13, rtol=1e-12)
            assert np.allclose(gv, dv[b, g, keys], atol=1e-13, rtol=1e-12)
