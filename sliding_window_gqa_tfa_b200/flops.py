"""Useful-work accounting for the throughput metric (host arithmetic only).

The metric counts 4*D flops per allowed (batch, query head, row, key) pair:
2*D for the q.k dot product and 2*D for the p*v accumulation.  Masked pairs
-- beyond the causal diagonal, outside the window, dropped by the key mask --
count nothing, even where a tile computes them.
"""
from __future__ import annotations

import numpy as np


def allowed_pairs(B, Hq, L, S, *, causal, window=0, key_mask=None) -> int:
    """Number of allowed (b, h, i, j) quadruples, in closed form per key."""
    P = S - L
    j = np.arange(S, dtype=np.int64)
    if causal:
        # key j is reachable from rows i with P + i >= j; with a window also P + i < j + window
        first_row = np.maximum(j - P, 0)
        last_row = np.full(S, L - 1, dtype=np.int64)
        if window > 0:
            last_row = np.minimum(last_row, j + window - 1 - P)
        reach = np.maximum(last_row - first_row + 1, 0)
    else:
        reach = np.full(S, L, dtype=np.int64)
    if key_mask is None:
        return int(reach.sum()) * B * Hq
    km = np.asarray(key_mask.cpu().numpy() if hasattr(key_mask, "cpu") else key_mask)
    keep = (km.reshape(B, S) > 0.5).astype(np.int64)
    return int((keep * reach[None, :]).sum()) * Hq


def useful_flops(B, Hq, L, S, D, *, causal, window=0, key_mask=None) -> int:
    return 4 * D * allowed_pairs(B, Hq, L, S, causal=causal, window=window, key_mask=key_mask)


def algorithmic_bytes(B, Hq, Hkv, L, S, D, *, key_mask=False) -> int:
    """Q read + O written once, K and V read once (bf16); key mask read once."""
    return 2 * D * (2 * B * Hq * L + 2 * B * Hkv * S) + (4 * B * S if key_mask else 0)


def workload_flops(w, key_mask=None) -> int:
    """Useful flops of one call on workload w (dense, rotating cache or packed
    variable-length): 4*D per allowed pair, summed per sequence for varlen."""
    if w.seqlens is not None:
        return sum(useful_flops(1, w.Hq, L, S, w.D, causal=w.causal, window=w.window)
                   for L, S in w.seqlens)
    f = useful_flops(w.B, w.Hq, w.L, w.S, w.D, causal=w.causal, window=w.window, key_mask=key_mask)
    # backward: five products of 2*D per allowed pair (S = Q K^T, dP = dO V^T,
    # dV = P^T dO, dQ = dS K, dK = dS^T Q) against the forward's two
    return f * 5 // 2 if w.backward else f


def workload_bytes(w) -> int:
    """Algorithmic bytes of one call: Q read and O written once, the K/V rows that
    exist read once (the ring's rows for a rotating cache), the key mask once."""
    if w.seqlens is not None:
        Tq = sum(L for L, _ in w.seqlens)
        Tk = sum(S for _, S in w.seqlens)
        return 2 * w.D * (2 * Tq * w.Hq + 2 * Tk * w.Hkv)
    S = min(w.S, w.ring_rows) if w.ring_rows else w.S
    fwd = algorithmic_bytes(w.B, w.Hq, w.Hkv, w.L, S, w.D, key_mask=w.key_mask_keep is not None)
    if w.backward:  # + dO read and dQ written, dK and dV written
        return fwd + 2 * w.D * (2 * w.B * w.Hq * w.L + 2 * w.B * w.Hkv * S)
    return fwd
