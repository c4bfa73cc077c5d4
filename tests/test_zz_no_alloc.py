"""tfa_prefill_noalloc: the entry point for callers that cannot allocate device
memory (their allocator owns it all, or allocating is not allowed where they
call).  It must give the same attention output as tfa_prefill, call after
call, while taking its scratch from the library's fixed device array instead
of allocating any.  This file is collected last on purpose: if it fails, a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02  # the operator tolerance every parity test here uses


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call(fn, w, dq, dk, dv, dkm, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(_ptr(dq), _ptr(dk), _ptr(dv), _ptr(out), w.B, w.Hq, w.Hkv, w.L, w.S, w.D,
            float(w.softmax_scale), int(w.causal), int(w.window), _ptr(dkm), stream)
    assert rc == tb.TFA_OK, f"{fn.__name__}: {tb.status_string(rc)} {tb.last_error()}"


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
    _call(tb.tfa_prefill, w, dq, dk, dv, dkm, ref)
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        out = torch.full_like(dq, float("nan"))
        _call(tb.tfa_prefill_noalloc, w, dq, dk, dv, dkm, out)
        assert tb.tfa_check_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == tb.TFA_OK
        got = out.float().cpu().numpy()
        exp = ref.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.all(np.abs(got - exp) <= ATOL + RTOL * np.abs(exp))


def test_noalloc_validates_like_tfa_prefill():
    w = shaped(1, 6, 4, 33, 47, 128)  # 6 % 4 != 0
    a = ctypes.c_void_p(0x10000)
    rc = tb.tfa_prefill_noalloc(a, a, a, a, w.B, w.Hq, w.Hkv, w.L, w.S, w.D, 0.1, 1, 0, None,
                                None)
    assert rc == tb.TFA_ERR_HEADS
