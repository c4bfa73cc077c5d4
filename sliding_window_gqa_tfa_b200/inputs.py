"""Seeded synthetic inputs for tiled GQA prefill attention.

This module is the ONE piece shared by the CUDA path's harness and the CPU
oracle's tests: it draws the arrays both sides consume and holds none of the
attention arithmetic.

Recipe: a CPU ``torch.Generator`` seeded with ``seed``; fp32 ``randn`` drawn in
the order Q, K, V (K multiplied by ``k_scale`` before the cast), then, when the
workload has a key mask, ``rand(B, S) >= 1 - keep`` as the 1/0 fp32 key mask,
then, when it has attention sinks, ``sink_scale * randn(Hq)`` fp32 sink logits;
then, for a backward workload, ``randn`` of q's shape as the upstream gradient
dO (bf16); Q/K/V are cast to bf16 (round to nearest even).  A logit softcap
is a plain number of the workload (Gemma-2 uses 50).  The shapes are the model
shapes the pages use: Qwen3-0.6B (16 query heads, 8 KV heads, head dim 128,
tiny-llm "Week 2 Day 5"), the Llama geometry of TensorFold PR 3269 (56 query
heads, 8 KV heads, group 7, head dim 128), the 1024-key sliding window of the
same PR and of mlx-lm PR 2006 (rotating cache: window - 1 + L keys per chunk),
and the 2048-token prefill chunks of mlx-lm PR 2006's benchmark.  No public
dataset is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    S: int
    D: int
    causal: bool = True
    window: int = 0
    key_mask_keep: float | None = None  # None: no key mask; else Bernoulli keep prob
    k_scale: float = 1.0
    scale: float | None = None  # None: 1/sqrt(D)
    softcap: float = 0.0        # 0: none
    sink_scale: float | None = None  # None: no sinks; else sinks ~ sink_scale * N(0, 1)
    # rotating cache: K/V hold ring_rows rows, position j in row j mod ring_rows
    ring_rows: int = 0
    # packed variable-length batch: ((L_b, S_b), ...) per sequence; B = len(seqlens),
    # L / S = the longest query / key count
    seqlens: tuple | None = None
    # the backward pass (gradients of q, k, v for an upstream gradient of the output)
    backward: bool = False
    # backward given the forward's output and per-row log-sum-exp (computed once,
    # before any timing, as a training step's forward would leave them)
    saved_stats: bool = False

    @property
    def kind(self) -> str:
        if self.backward:
            return "backward"
        return "varlen" if self.seqlens is not None else "ring" if self.ring_rows else "dense"

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    @property
    def prefix(self) -> int:
        return self.S - self.L

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Prompt lengths of the variable-length workload (a fixed draw, uniform in [256, 4096]).
_VARLEN16 = (3184, 1291, 2869, 417, 3977, 2050, 733, 1504, 256, 3511, 1876, 988, 4096, 2290, 612, 1362)
_VARLEN16_MAX = max(_VARLEN16)

WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    # 33 query rows over 47 keys (prefix 14): crosses both tile tails.
    Workload("witness_33x47", B=1, Hq=8, Hkv=2, L=33, S=47, D=128),
    # Qwen3-0.6B attention geometry, batch 4, 2048-token prompt, no prefix.
    Workload("qwen3_prefill_b4_2048", B=4, Hq=16, Hkv=8, L=2048, S=2048, D=128),
    # Llama GQA chunk: 2048 new rows over 8192 keys (prefix 6144), group 7.
    Workload("llama_gqa_chunk_2048x8192", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128),
    Workload("llama_gqa_chunk_2048x8192_keymask", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128,
             key_mask_keep=0.9),
    # Rotating-cache sliding window: 1024-key window, chunk 2048, S = 1023 + 2048.
    Workload("swa_rotating_w1024_2048", B=1, Hq=32, Hkv=8, L=2048, S=3071, D=128, window=1024),
    # Long-context chunk at 32K keys, K scaled x4 to sharpen the softmax.
    Workload("long_chunk_2048x32768", B=1, Hq=32, Hkv=8, L=2048, S=32768, D=128, k_scale=4.0),
    Workload("long_chunk_2048x32768_d64", B=1, Hq=32, Hkv=8, L=2048, S=32768, D=64, k_scale=4.0),
    Workload("bidirectional_4096", B=1, Hq=32, Hkv=8, L=4096, S=4096, D=128, causal=False,
             k_scale=4.0),
    # Score variants on the Llama chunk: a Gemma-2 style logit softcap (50, with K
    # scaled x4 so that the cap bends the scores) and per-head attention sinks.
    Workload("llama_gqa_chunk_2048x8192_softcap50", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128,
             k_scale=4.0, softcap=50.0),
    Workload("llama_gqa_chunk_2048x8192_sinks", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128,
             sink_scale=2.0),
    # Rotating cache of TensorFold's sliding layer (WINDOW 1024, RING 1088): 16
    # sequences 32K tokens in, a 64-row chunk each, and 64 sequences decoding.
    Workload("swa_ring_r1088_chunk64_b16", B=16, Hq=32, Hkv=8, L=64, S=32768, D=128, window=1024,
             ring_rows=1088),
    Workload("swa_ring_r1088_decode_b64", B=64, Hq=32, Hkv=8, L=1, S=32768, D=128, window=1024,
             ring_rows=1088),
    # Packed variable-length prefill of 16 Qwen3-shaped prompts (256..4096 tokens).
    Workload("varlen_qwen3_16seqs", B=16, Hq=16, Hkv=8, L=_VARLEN16_MAX, S=_VARLEN16_MAX, D=128,
             seqlens=tuple((n, n) for n in _VARLEN16)),
    # The backward pass on the Llama chunk (gradients of q, k, v).
    Workload("llama_gqa_chunk_2048x8192_backward", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128,
             backward=True),
    # The same backward from the forward's saved output and log-sum-exp.
    Workload("llama_gqa_chunk_2048x8192_backward_saved", B=1, Hq=56, Hkv=8, L=2048, S=8192, D=128,
             backward=True, saved_stats=True),
    # Short queries (1 <= L <= 8): token-by-token decoding over a long cache,
    # batched Qwen3-shaped decoding, and an 8-row chunk (e.g. draft verification).
    Workload("llama_gqa_decode_1x32768", B=1, Hq=56, Hkv=8, L=1, S=32768, D=128),
    Workload("qwen3_decode_b16_8192", B=16, Hq=16, Hkv=8, L=1, S=8192, D=128),
    Workload("llama_gqa_chunk_8x8192_b4", B=4, Hq=56, Hkv=8, L=8, S=8192, D=128),
    Workload("llama_gqa_decode_1x32768_sinks_softcap", B=1, Hq=56, Hkv=8, L=1, S=32768, D=128,
             softcap=30.0, sink_scale=2.0),
]}

# The workload the throughput figure is quoted on.
HEADLINE = "llama_gqa_chunk_2048x8192"


def make_inputs(w: Workload, seed: int = 0):
    """Return (q, k, v, key_mask) as CPU tensors: bf16 [B,Hq,L,D], bf16 [B,Hkv,S,D] x2,
    and fp32 [B,S] (or None).  A rotating-cache workload's k/v are the ring contents
    [B,Hkv,ring_rows,D]; a variable-length workload's are packed: q [sum L_b, Hq, D],
    k/v [sum S_b, Hkv, D] (see varlen_cu).  Sink logits, when the workload has
    them, come from make_sinks with the same seed."""
    return _draw(w, seed)[:4]


def varlen_cu(w: Workload):
    """int32 prefix sums (cu_seqlens_q, cu_seqlens_k) of a variable-length workload."""
    import numpy as np

    cq = np.concatenate([[0], np.cumsum([L for L, _ in w.seqlens])]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum([S for _, S in w.seqlens])]).astype(np.int32)
    return cq, ck


def make_sinks(w: Workload, seed: int = 0):
    """fp32 [Hq] sink logits of the workload (drawn after q, k, v and the key
    mask from the same generator), or None."""
    return _draw(w, seed)[4]


def _draw(w: Workload, seed: int):
    g = torch.Generator().manual_seed(seed)
    if w.seqlens is not None:
        q_shape = (sum(L for L, _ in w.seqlens), w.Hq, w.D)
        kv_shape = (sum(S for _, S in w.seqlens), w.Hkv, w.D)
    else:
        q_shape = (w.B, w.Hq, w.L, w.D)
        kv_shape = (w.B, w.Hkv, w.ring_rows if w.ring_rows else w.S, w.D)
    q = torch.randn(*q_shape, generator=g, dtype=torch.float32)
    k = torch.randn(*kv_shape, generator=g, dtype=torch.float32)
    v = torch.randn(*kv_shape, generator=g, dtype=torch.float32)
    if w.k_scale != 1.0:
        k = k * w.k_scale
    key_mask = None
    if w.key_mask_keep is not None:
        key_mask = (torch.rand(w.B, w.S, generator=g) >= (1.0 - w.key_mask_keep)).float()
    sinks = None
    if w.sink_scale is not None:
        sinks = w.sink_scale * torch.randn(w.Hq, generator=g, dtype=torch.float32)
    dout = None
    if w.backward:
        dout = torch.randn(*q_shape, generator=g, dtype=torch.float32).bfloat16()
    return q.bfloat16(), k.bfloat16(), v.bfloat16(), key_mask, sinks, dout


def make_dout(w: Workload, seed: int = 0):
    """bf16 upstream gradient of the output (shape of q) of a backward workload,
    drawn after q, k, v, the key mask and the sinks from the same generator."""
    return _draw(w, seed)[5]


def sample_rows(w: Workload, n_per_head: int = 24, seed: int = 0):
    """Flat row indices (b * Hq + h) * L + i of a full-size dense workload to
    check one by one: the tile edges and tails, the middle row and random rows,
    n_per_head of them in every head."""
    import numpy as np

    rng = np.random.default_rng(seed)
    L = w.L
    n_per_head = min(n_per_head, L)  # a short query has fewer rows than the sample size
    fixed = [0, 1, 127, 128, 255, 256, L // 2, L - 129, L - 128, L - 2, L - 1]
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            pick = set(i for i in fixed if 0 <= i < L)
            while len(pick) < n_per_head:
                pick.add(int(rng.integers(0, L)))
            rows += [(b * w.Hq + h) * L + i for i in sorted(pick)]
    return np.array(rows, dtype=np.int64)


def shaped(B, Hq, Hkv, L, S, D, *, causal=True, window=0, key_mask_keep=None, k_scale=1.0,
           softcap=0.0, sink_scale=None, name="custom") -> Workload:
    """A workload of arbitrary shape drawn by the same recipe (for edge-case tests)."""
    return Workload(name, B=B, Hq=Hq, Hkv=Hkv, L=L, S=S, D=D, causal=causal, window=window,
                    key_mask_keep=key_mask_keep, k_scale=k_scale, softcap=softcap,
                    sink_scale=sink_scale)
