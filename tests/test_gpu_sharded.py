"""One call's (batch, KV group) units shared by ranks, run on one GPU.

sliding_window_gqa_tfa_b200.dist gives rank r a contiguous range of the B*Hkv
units and runs it as at most three ordinary library calls on slices of the
tensors (the tail groups of one element, whole elements, the head groups of
one element), the key-mask rows and sink logits sliced alike.  Here every
rank's share runs in turn on the same GPU into one output buffer -- no
collective is involved -- and the whole output must match the fp64 oracle,
with each rank writing exactly its own query planes.
"""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import dist as tdist
from sliding_window_gqa_tfa_b200.inputs import make_inputs, make_sinks, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02


@pytest.mark.parametrize("world,w", [
    (2, shaped(1, 8, 4, 300, 700, 128, name="b1_hkv4")),
    (3, shaped(2, 6, 3, 200, 450, 64, window=129, key_mask_keep=0.8, name="b2_hkv3_window_mask")),
    (4, shaped(3, 8, 2, 40, 90, 128, causal=False, name="b3_hkv2_packed_bidirectional")),
    (5, shaped(2, 12, 4, 140, 300, 128, sink_scale=2.0, name="b2_hkv4_sinks")),
], ids=lambda x: x if isinstance(x, int) else x.name)
def test_every_rank_share_on_one_gpu_equals_the_whole_call(world, w):
    q, k, v, km = make_inputs(w, seed=31)
    sinks = make_sinks(w, seed=31)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dkm = km.cuda() if km is not None else None
    dsinks = sinks.cuda() if sinks is not None else None
    out = torch.full_like(dq, float("nan"))
    planes = out.view(w.B * w.Hq, -1)
    for rank in range(world):
        before = planes.clone()
        tdist.sharded_prefill(dq, dk, dv, out, world, rank, key_mask=dkm, scale=w.softmax_scale,
                              causal=w.causal, window=w.window, sinks=dsinks)
        torch.cuda.synchronize()
        p0, p1 = tdist.rank_planes(w.B, w.Hq, w.Hkv, world, rank)
        changed = (planes != before) & ~(torch.isnan(planes) & torch.isnan(before))
        rows_changed = changed.any(dim=1).nonzero().flatten().tolist()
        assert all(p0 <= r_ < p1 for r_ in rows_changed)  # only this rank's planes
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km, sinks=sinks)
    got = out.float().cpu().double().numpy()
    assert np.all(np.isfinite(got))  # every plane was written by some rank
    assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))
