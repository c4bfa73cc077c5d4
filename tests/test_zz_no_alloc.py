"""tfa_prefill_noalloc: the entry point for callers that cannot allocate device
memory (their allocator owns it all, or allocating is not allowed where they
call).  Call after call it must give the same attention output as
tfa_prefill, within the operator tolerance, and match the fp64 definition
element by element, while taking its scratch from the library's fixed device
array instead of allocating any.  This file is collected last on purpose: if
it fails, a run that stops at the first failure has already run every other
test.  Nothing else in the test suite calls this entry point, so the first
test below is the process's first no-alloc call, alone or after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02  # the operator tolerance every parity test here uses


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call(fn, w, dq, dk, dv, dkm, out, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return fn(_ptr(dq), _ptr(dk), _ptr(dv), _ptr(out), w.B, w.Hq, w.Hkv, w.L, w.S, w.D,
              float(w.softmax_scale), int(w.causal), int(w.window), _ptr(dkm),
              ctypes.c_void_p(s.cuda_stream))


def _ok(rc, fn):
    assert rc == tb.TFA_OK, f"{fn.__name__}: {tb.status_string(rc)} {tb.last_error()}"


def test_first_noalloc_call_under_capture_is_refused():
    # the first call on a device clears the static array with a memset, which a
    # stream capture would record instead of running: it is refused instead
    w = WORKLOADS["witness_33x47"]
    q, k, v, _ = make_inputs(w, seed=5)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(dq)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        rc = _call(tb.tfa_prefill_noalloc, w, dq, dk, dv, None, out, stream=s)
    assert rc == tb.TFA_ERR_CAPTURE
    del g
    torch.cuda.synchronize()


@pytest.mark.parametrize("w", [
    WORKLOADS["witness_33x47"],
    shaped(1, 8, 2, 300, 700, 128, window=129, key_mask_keep=0.8, name="window_keymask"),
    shaped(2, 4, 2, 130, 300, 64, causal=False, name="d64_bidirectional"),
], ids=lambda w: w.name)
def test_noalloc_matches_tfa_prefill_on_consecutive_calls(w):
    assert torch.cuda.is_available()
    q, k, v, km = make_inputs(w, seed=3)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dkm = km.cuda() if km is not None else None
    ref = torch.empty_like(dq)
    _ok(_call(tb.tfa_prefill, w, dq, dk, dv, dkm, ref), tb.tfa_prefill)
    exact = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                             key_mask=km)
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        out = torch.full_like(dq, float("nan"))
        _ok(_call(tb.tfa_prefill_noalloc, w, dq, dk, dv, dkm, out), tb.tfa_prefill_noalloc)
        assert tb.tfa_check_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == tb.TFA_OK
        got = out.float().cpu().double().numpy()
        exp = ref.float().cpu().double().numpy()
        assert np.all(np.isfinite(got))
        # against tfa_prefill (another schedule, so another rounding order)
        assert np.all(np.abs(got - exp) <= ATOL + RTOL * np.abs(exp))
        # against the fp64 definition, element by element
        assert np.all(np.abs(got - exact) <= ATOL + RTOL * np.abs(exact))


def test_noalloc_validates_like_tfa_prefill():
    w = shaped(1, 6, 4, 33, 47, 128)  # 6 % 4 != 0
    a = ctypes.c_void_p(0x10000)
    rc = tb.tfa_prefill_noalloc(a, a, a, a, w.B, w.Hq, w.Hkv, w.L, w.S, w.D, 0.1, 1, 0, None,
                                None)
    assert rc == tb.TFA_ERR_HEADS
