"""CUDA-graph capture of the attention calls, checked against the fp64 oracle.

The decode case is the fixed-capacity masked form of short-query attention:
the key/value cache keeps a fixed capacity S, the key mask marks the slots a
sequence has filled, and one captured graph is replayed as the cache fills
(the pages route short queries over a growing cache through a separate
decode path; here the same captured call serves every length).  Each replay
rewrites the inputs in place and must match the oracle on the new data, which
also shows that the split schedule's cross-CTA handshake does not depend on
anything frozen into the graph."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


def _assert_close(got, ref, what):
    got = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), what
    bad = np.abs(got - ref) > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements off, max err {np.abs(got - ref).max():.3g}"


def _length_mask(B, S, lengths):
    j = torch.arange(S)
    return torch.stack([(j < n).float() for n in lengths])


def test_decode_graph_fixed_capacity_cache():
    w = shaped(2, 14, 2, 1, 8192, 128)  # 2 KV groups of 7 heads per sequence: split over all SMs
    s = torch.cuda.Stream()
    q0, k0, v0, _ = make_inputs(w, seed=100)
    q_s, k_s, v_s = q0.cuda(), k0.cuda(), v0.cuda()
    m_s = _length_mask(w.B, w.S, [w.S, w.S]).cuda()
    o_s = torch.empty_like(q_s)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):  # the stream's first call creates its scratch, outside capture
        tb.prefill(q_s, k_s, v_s, scale=w.softmax_scale, causal=True, key_mask=m_s, out=o_s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tb.prefill(q_s, k_s, v_s, scale=w.softmax_scale, causal=True, key_mask=m_s, out=o_s)
    s.synchronize()
    for step, lengths in enumerate([(100, 5000), (4097, 8192), (1, 2), (8191, 6000), (8192, 128)]):
        q, k, v, _ = make_inputs(w, seed=200 + step)
        km = _length_mask(w.B, w.S, lengths)
        with torch.cuda.stream(s):
            q_s.copy_(q)
            k_s.copy_(k)
            v_s.copy_(v)
            m_s.copy_(km)
            o_s.fill_(float("nan"))
            g.replay()
        s.synchronize()
        tb.check_status(s)
        ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, key_mask=km)
        _assert_close(o_s.reshape(-1, w.D), ref.reshape(-1, w.D), f"replay {step} lengths {lengths}")
    # a direct call on the same stream after the replays still sees a fresh handshake
    q, k, v, _ = make_inputs(w, seed=300)
    km = _length_mask(w.B, w.S, (3000, 7))
    with torch.cuda.stream(s):
        o = tb.prefill(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=True,
                       key_mask=km.cuda())
    s.synchronize()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, key_mask=km)
    _assert_close(o.reshape(-1, w.D), ref.reshape(-1, w.D), "direct call after replays")
    del g


def test_prefill_graph_split_schedule_replays():
    w = shaped(1, 8, 2, 300, 5000, 128)
    s = torch.cuda.Stream()
    q0, k0, v0, _ = make_inputs(w, seed=400)
    q_s, k_s, v_s = q0.cuda(), k0.cuda(), v0.cuda()
    o_s = torch.empty_like(q_s)
    flags = tb.TFA_DEBUG_FORCE_SPLIT
    with torch.cuda.stream(s):
        tb.prefill(q_s, k_s, v_s, scale=w.softmax_scale, causal=True, out=o_s, debug_flags=flags)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tb.prefill(q_s, k_s, v_s, scale=w.softmax_scale, causal=True, out=o_s, debug_flags=flags)
    s.synchronize()
    for step in range(3):
        q, k, v, _ = make_inputs(w, seed=500 + step)
        with torch.cuda.stream(s):
            q_s.copy_(q)
            k_s.copy_(k)
            v_s.copy_(v)
            o_s.fill_(float("nan"))
            g.replay()
        s.synchronize()
        tb.check_status(s)
        ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True)
        _assert_close(o_s.reshape(-1, w.D), ref.reshape(-1, w.D), f"prefill replay {step}")
    del g


def test_first_call_under_capture_is_refused():
    w = shaped(1, 8, 2, 1, 1000, 128)
    q, k, v, _ = make_inputs(w, seed=600)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(dq)
    torch.cuda.synchronize()
    # a stream the library has never seen (torch's pooled streams are reused,
    # so create a fresh one)
    from cuda.bindings import runtime as rt
    err, raw = rt.cudaStreamCreate()
    assert err == rt.cudaError_t.cudaSuccess
    s = torch.cuda.ExternalStream(int(raw))
    g = torch.cuda.CUDAGraph()
    with pytest.raises(tb.TfaError) as e:
        with torch.cuda.graph(g, stream=s):
            tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, out=out)
    assert e.value.code == tb.TFA_ERR_CAPTURE
    del g
    torch.cuda.synchronize()
    # outside capture the same stream then works
    with torch.cuda.stream(s):
        tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, out=out)
    s.synchronize()
    rt.cudaStreamDestroy(raw)
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True)
    _assert_close(out.reshape(-1, w.D), ref.reshape(-1, w.D), "after refused capture")
