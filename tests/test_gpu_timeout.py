"""The kernel's give-up path, run on purpose without faulting or hanging the GPU.

Every pipeline wait of the kernel is bounded; a wait that runs out raises the
CTA's abort flag, records a timeout in the device status word, and the CTA
drains its in-flight TMA copies and tensor-core work before it frees tensor
memory and exits.  TFA_DEBUG_SHORT_WAITS gives the waits a limit of ~1000 SM
cycles, far below the first TMA load's latency, so the waits run out on an
ordinary call (no flag that nothing sets, no bad address, no trap).  The call
must report TFA_ERR_TIMEOUT, and the next ordinary call on the same stream must
be correct: the status word was cleared, and the split schedule's ready flags
belong to an epoch that advanced past the aborted launch.
"""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


def _close(got, ref):
    got = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))


@pytest.mark.parametrize("L,S,flags", [
    (300, 700, 0), (300, 700, tb.TFA_DEBUG_FORCE_SPLIT), (300, 700, tb.TFA_DEBUG_NO_SPLIT),
    (33, 4000, 0), (33, 4000, tb.TFA_DEBUG_FORCE_SPLIT),
], ids=["default", "split", "whole_items", "packed", "packed_split"])
def test_short_waits_give_up_and_the_next_call_is_clean(L, S, flags):
    # L = 300: 128-row query tiles; L = 33: packed tiles (up to three of a KV
    # group's four query heads per tile), whose split key ranges end in the
    # merge that both softmax warpgroups share
    w = shaped(1, 8, 2, L, S, 128)
    q, k, v, _ = make_inputs(w, seed=21)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True)
    s = torch.cuda.current_stream()
    out = torch.empty_like(dq)
    tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, out=out)  # stream set-up
    tb.check_status(s)
    with pytest.raises(tb.TfaError) as e:
        tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, out=out,
                   debug_flags=flags | tb.TFA_DEBUG_SHORT_WAITS | tb.TFA_DEBUG_SYNC)
    assert e.value.code == tb.TFA_ERR_TIMEOUT
    # the status word was read and cleared by that call
    tb.check_status(s)
    for _ in range(2):
        out = torch.full_like(dq, float("nan"))
        tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True, out=out, debug_flags=flags)
        tb.check_status(s)
        _close(out, ref)
