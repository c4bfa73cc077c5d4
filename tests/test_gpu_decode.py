"""GPU parity of tfa_decode (1 <= L <= 8 query rows; L = 1 is token-by-token
decoding) against the fp64 oracle: same definition, same tolerance
(atol = rtol = 0.02 on the bf16 output) as the prefill path."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import make_inputs, shaped

pytestmark = pytest.mark.gpu

ATOL = RTOL = 0.02

CASES = [
    ("l1_g7", shaped(1, 56, 8, 1, 4096, 128)),
    ("l1_g4_b3", shaped(3, 16, 4, 1, 700, 128)),
    ("l2_g2", shaped(2, 8, 4, 2, 333, 128)),
    ("l7_g7", shaped(1, 14, 2, 7, 1000, 128)),
    ("l8_g16_chunks", shaped(1, 32, 2, 8, 2000, 128)),      # 16 heads x 8 rows > 128: two tiles per group
    ("l8_mha", shaped(2, 4, 4, 8, 257, 128)),
    ("l1_window", shaped(1, 8, 2, 1, 5000, 128, window=1024)),
    ("l4_window_short", shaped(1, 8, 2, 4, 300, 128, window=3)),
    ("l3_keymask", shaped(2, 8, 2, 3, 900, 128, key_mask_keep=0.5)),
    ("l1_keymask_sparse", shaped(1, 8, 2, 1, 3000, 128, key_mask_keep=0.02)),
    ("l5_bidirectional", shaped(1, 8, 2, 5, 777, 128, causal=False)),
    ("l1_long_split", shaped(1, 8, 8, 1, 65536, 128, k_scale=4.0)),
    ("l1_min_keys", shaped(1, 4, 2, 1, 1, 128)),
    ("l8_min_keys", shaped(1, 4, 2, 8, 8, 128)),
    ("d64_l1", shaped(2, 16, 8, 1, 1500, 64)),
    ("d64_l6_window_mask", shaped(1, 12, 4, 6, 2500, 64, window=500, key_mask_keep=0.8)),
]


@pytest.mark.parametrize("name,w", CASES, ids=[n for n, _ in CASES])
def test_decode_parity(name, w):
    q, k, v, km = make_inputs(w, seed=21)
    o = tb.prefill(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=w.causal,
                   window=w.window, key_mask=km.cuda() if km is not None else None)
    tb.check_status()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                           key_mask=km)
    got = o.float().cpu().double().numpy()
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{name}: {bad.sum()} out of tolerance, max abs err {err.max():.4g}"
    print(f"{name}: max abs err {err.max():.3e}")


def test_decode_fully_masked_rows_are_zero_and_stream_order_holds():
    w = shaped(2, 8, 2, 1, 500, 128)
    q, k, v, _ = make_inputs(w, seed=22)
    km = torch.ones(2, 500)
    km[1] = 0
    o = tb.prefill(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=True,
                   key_mask=km.cuda())
    tb.check_status()
    assert torch.all(o[1] == 0).item()
    ref = oracle.attention(q, k, v, scale=w.softmax_scale, causal=True, key_mask=km)
    assert np.allclose(o[0].float().cpu().numpy(), ref[0], atol=ATOL, rtol=RTOL)


def test_decode_matches_the_last_rows_of_a_prefill():
    """Decoding the last L rows equals those rows of a longer prefill chunk
    over the same keys (the chunked-prefix identity, across the two paths)."""
    w = shaped(1, 16, 4, 64, 1000, 128)
    q, k, v, _ = make_inputs(w, seed=23)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    full = tb.prefill(dq, dk, dv, scale=w.softmax_scale, causal=True)
    for L in (1, 5, 8):
        part = tb.prefill(dq[:, :, -L:].contiguous(), dk, dv, scale=w.softmax_scale, causal=True)
        tb.check_status()
        a = part.float().cpu().numpy()
        b = full[:, :, -L:].float().cpu().numpy()
        assert np.allclose(a, b, atol=ATOL, rtol=RTOL)
