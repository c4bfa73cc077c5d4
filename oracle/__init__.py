"""fp64 CPU oracle for tiled GQA prefill attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it and shares no code with it.

The arithmetic lives in ``tfa_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only builds it with gcc, marshals arrays through ctypes and
returns numpy float64 results.  See the C file's header for the definition
and the passages of the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tfa_oracle.c")
_LIB = os.path.join(_HERE, "libtfa_oracle.so")
_lock = threading.Lock()
_lib = None

# Planted mistakes understood by attention_mutant(); see tfa_oracle.c.
MUTATIONS = {
    "causal_sees_next": 1,
    "window_one_wider": 2,
    "head_modulo": 3,
    "no_prefix_offset": 4,
    "drop_scale": 5,
    "keymask_inverted": 6,
    "empty_row_uniform": 7,
    "softcap_before_scale": 8,
    "sink_scaled": 9,
    "sink_in_numerator": 10,
}
# Planted mistakes of the rotating-cache and packed variable-length entry points.
RING_MUTATIONS = {"ring_slot_shifted": 11}
VARLEN_MUTATIONS = {"varlen_packed_causal": 12, "head_modulo": 3, "no_prefix_offset": 4}
BACKWARD_MUTATIONS = {"bwd_no_delta": 13, "bwd_dk_no_scale": 14, "bwd_dq_uses_v": 15,
                      "head_modulo": 3, "causal_sees_next": 1, "keymask_inverted": 6}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (portable flags: no -march=native, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_attention.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f64,
                                             i32, i32, P, P, i64, i32]
            lib.oracle_attention.restype = i32
            lib.oracle_attention_ex.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f64,
                                                i32, i32, P, f64, P, P, i64, i32]
            lib.oracle_attention_ex.restype = i32
            lng = ctypes.c_long
            lib.oracle_attention_mutant.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, lng, i32,
                                                    f64, i32, i32, P, f64, P, i32]
            lib.oracle_attention_ring.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, lng, i32,
                                                  f64, i32, f64, P, P, i64, i32]
            lib.oracle_attention_ring.restype = i32
            lib.oracle_attention_varlen.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, f64,
                                                    i32, i32, f64, P, i32]
            lib.oracle_attention_varlen.restype = i32
            lib.oracle_attention_varlen_mutant.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32,
                                                           f64, i32, i32, i32]
            lib.oracle_attention_varlen_mutant.restype = i32
            lib.oracle_attention_backward.argtypes = [P] * 7 + [i32] * 6 + [f64, i32, i32, P, i32]
            lib.oracle_attention_backward.restype = i32
            lib.oracle_attention_backward_mutant.argtypes = [P] * 7 + [i32] * 6 + [f64, i32, i32, P,
                                                                                 i32]
            lib.oracle_attention_backward_mutant.restype = i32
            lib.oracle_attention_backward_dq_rows.argtypes = [P] * 5 + [i32] * 6 + [f64, i32, i32, P,
                                                                                  P, i64, i32]
            lib.oracle_attention_backward_dq_rows.restype = i32
            lib.oracle_attention_backward_kv_rows.argtypes = [P] * 6 + [i32] * 6 + [f64, i32, i32, P,
                                                                                  i32, i32, P, i64,
                                                                                  i32]
            lib.oracle_attention_backward_kv_rows.restype = i32
            lib.oracle_attention_mutant.restype = i32
            lib.oracle_softmax_weights.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64,
                                                   i32, i32, P, i32, i32, i32]
            lib.oracle_softmax_weights.restype = i32
            lib.oracle_count_pairs.argtypes = [i32, i32, i32, i32, i32, i32, P]
            lib.oracle_count_pairs.restype = i64
            lib.oracle_allowed.argtypes = [ctypes.c_long] * 4 + [i32, ctypes.c_long, P]
            lib.oracle_allowed.restype = i32
            lib.oracle_attention_blockwise.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32,
                                                       f64, i32, i32, P, i32, i32, i32, P]
            lib.oracle_attention_blockwise.restype = i32
            _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch

    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _mask(m):
    if m is None:
        return None
    if not isinstance(m, np.ndarray):
        m = m.detach().cpu().float().numpy()
    return np.ascontiguousarray(m, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _shape(q, k):
    B, Hq, L, D = q.shape
    Bk, Hkv, S, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("q/k shapes disagree")
    return B, Hq, Hkv, L, S, D


def _sinks(sinks, Hq):
    if sinks is None:
        return None
    if not isinstance(sinks, np.ndarray):
        sinks = sinks.detach().cpu().float().numpy()
    sinks = np.ascontiguousarray(sinks, dtype=np.float32).reshape(-1)
    if sinks.size != Hq:
        raise ValueError("sinks must hold one logit per query head")
    return sinks


def attention(q, k, v, *, scale, causal, window=0, key_mask=None, softcap=0.0, sinks=None,
              rows=None, threads=0):
    """Plain fp64 definition.  softcap: 0 = none; sinks: fp32 [Hq] logits or None;
    rows: optional flattened (b*Hq+h)*L+i indices."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    sk = _sinks(sinks, Hq)
    if rows is None:
        out = np.empty((B, Hq, L, D), dtype=np.float64)
        r_ptr, nr = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((r.size, D), dtype=np.float64)
        r_ptr, nr = r.ctypes.data_as(ctypes.c_void_p), r.size
    rc = _load().oracle_attention_ex(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, Hq, Hkv, L, S,
                                     D, float(scale), int(bool(causal)), int(window), _ptr(km),
                                     float(softcap), _ptr(sk), r_ptr, nr, int(threads))
    if rc:
        raise ValueError(f"oracle_attention rejected its arguments (code {rc})")
    return out


def attention_mutant(q, k, v, *, scale, causal, window=0, key_mask=None, softcap=0.0,
                     sinks=None, mutation):
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    sk = _sinks(sinks, Hq)
    out = np.empty((B, Hq, L, D), dtype=np.float64)
    code = MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)
    rc = _load().oracle_attention_mutant(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, Hq, Hkv, L,
                                         S, 0, D, float(scale), int(bool(causal)), int(window),
                                         _ptr(km), float(softcap), _ptr(sk), code)
    if rc:
        raise ValueError(f"oracle_attention_mutant rejected its arguments (code {rc})")
    return out


def attention_ring(q, k_ring, v_ring, *, S, scale, window, softcap=0.0, sinks=None, rows=None,
                   threads=0, mutation=0):
    """Rotating cache: k/v [B,Hkv,R,D], key position j (0 <= j < S) in row j mod R;
    causal with a window, R >= window - 1 + L.  Returns [B,Hq,L,D] (or rows x D)."""
    qb, kb, vb = _bits(q), _bits(k_ring), _bits(v_ring)
    B, Hq, L, D = qb.shape
    Bk, Hkv, R, Dk = kb.shape
    if Bk != B or Dk != D:
        raise ValueError("q/k shapes disagree")
    sk = _sinks(sinks, Hq)
    code = RING_MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)
    if code:
        if rows is not None:
            raise ValueError("mutants compute every row")
        out = np.empty((B, Hq, L, D), dtype=np.float64)
        rc = _load().oracle_attention_mutant(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, Hq, Hkv,
                                             L, int(S), int(R), D, float(scale), 1, int(window),
                                             None, float(softcap), _ptr(sk), code)
    else:
        if rows is None:
            out = np.empty((B, Hq, L, D), dtype=np.float64)
            r_ptr, nr = None, 0
        else:
            r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            out = np.empty((r.size, D), dtype=np.float64)
            r_ptr, nr = r.ctypes.data_as(ctypes.c_void_p), r.size
        rc = _load().oracle_attention_ring(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, Hq, Hkv, L,
                                           int(S), int(R), D, float(scale), int(window),
                                           float(softcap), _ptr(sk), r_ptr, nr, int(threads))
    if rc:
        raise ValueError(f"oracle_attention_ring rejected its arguments (code {rc})")
    return out


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, *, scale, causal, window=0,
                     softcap=0.0, sinks=None, threads=0, mutation=0):
    """Packed variable-length attention: q [Tq,Hq,D], k/v [Tk,Hkv,D], int32 prefix sums
    cu_seqlens_* [B+1].  Returns [Tq,Hq,D] float64."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    Tq, Hq, D = qb.shape
    Tk, Hkv, Dk = kb.shape
    if Dk != D or vb.shape != kb.shape:
        raise ValueError("q/k/v shapes disagree")
    cq = np.ascontiguousarray(np.asarray(cu_seqlens_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int32))
    B = cq.size - 1
    if ck.size != B + 1 or cq[-1] != Tq or ck[-1] != Tk:
        raise ValueError("cu_seqlens must be [B+1] prefix sums ending at the packed lengths")
    sk = _sinks(sinks, Hq)
    out = np.empty((Tq, Hq, D), dtype=np.float64)
    code = VARLEN_MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)
    if code:
        rc = _load().oracle_attention_varlen_mutant(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out),
                                                    _ptr(cq), _ptr(ck), B, Hq, Hkv, D, float(scale),
                                                    int(bool(causal)), int(window), code)
    else:
        rc = _load().oracle_attention_varlen(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), _ptr(cq),
                                             _ptr(ck), B, Hq, Hkv, D, float(scale),
                                             int(bool(causal)), int(window), float(softcap),
                                             _ptr(sk), int(threads))
    if rc:
        raise ValueError(f"oracle_attention_varlen rejected its arguments (code {rc})")
    return out


def attention_backward(q, k, v, dout, *, scale, causal, window=0, key_mask=None, threads=0,
                       mutation=0):
    """Gradients (dq [B,Hq,L,D], dk, dv [B,Hkv,S,D], float64) of the plain definition
    for the upstream gradient dout [B,Hq,L,D] (bf16)."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    if db.shape != qb.shape or vb.shape != kb.shape:
        raise ValueError("dout must match q, v must match k")
    km = _mask(key_mask)
    dq = np.empty(qb.shape, dtype=np.float64)
    dk = np.empty(kb.shape, dtype=np.float64)
    dv = np.empty(kb.shape, dtype=np.float64)
    code = BACKWARD_MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)
    args = (_ptr(qb), _ptr(kb), _ptr(vb), _ptr(db), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, L, S,
            D, float(scale), int(bool(causal)), int(window), _ptr(km))
    rc = (_load().oracle_attention_backward_mutant(*args, code) if code
          else _load().oracle_attention_backward(*args, int(threads)))
    if rc:
        raise ValueError(f"oracle_attention_backward rejected its arguments (code {rc})")
    return dq, dk, dv


def attention_backward_dq_rows(q, k, v, dout, rows, *, scale, causal, window=0, key_mask=None,
                               threads=0):
    """dQ (float64, len(rows) x D) of the listed flattened rows (b*Hq+h)*L+i only."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((r.size, D), dtype=np.float64)
    rc = _load().oracle_attention_backward_dq_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(db), _ptr(out),
                                                   B, Hq, Hkv, L, S, D, float(scale),
                                                   int(bool(causal)), int(window), _ptr(km),
                                                   r.ctypes.data_as(ctypes.c_void_p), r.size,
                                                   int(threads))
    if rc:
        raise ValueError(f"oracle_attention_backward_dq_rows rejected its arguments (code {rc})")
    return out


def attention_backward_kv_rows(q, k, v, dout, *, b, g, keys, scale, causal, window=0,
                               key_mask=None, threads=0):
    """(dk, dv) float64 (len(keys) x D each) of the listed keys of KV head g, batch b."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    kk = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    dk = np.empty((kk.size, D), dtype=np.float64)
    dv = np.empty((kk.size, D), dtype=np.float64)
    rc = _load().oracle_attention_backward_kv_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(db), _ptr(dk),
                                                   _ptr(dv), B, Hq, Hkv, L, S, D, float(scale),
                                                   int(bool(causal)), int(window), _ptr(km), int(b),
                                                   int(g), kk.ctypes.data_as(ctypes.c_void_p),
                                                   kk.size, int(threads))
    if rc:
        raise ValueError(f"oracle_attention_backward_kv_rows rejected its arguments (code {rc})")
    return dk, dv


def attention_blockwise(q, k, v, *, scale, causal, window=0, key_mask=None, bq=128, bk=128,
                        skip_empty=True):
    """Tiled online-softmax variant; returns (output, key tiles visited per row block sum)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    out = np.empty((B, Hq, L, D), dtype=np.float64)
    visited = ctypes.c_int64(0)
    rc = _load().oracle_attention_blockwise(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, Hq, Hkv,
                                            L, S, D, float(scale), int(bool(causal)), int(window),
                                            _ptr(km), int(bq), int(bk), int(bool(skip_empty)),
                                            ctypes.byref(visited))
    if rc:
        raise ValueError(f"oracle_attention_blockwise rejected its arguments (code {rc})")
    return out, int(visited.value)


def softmax_weights(q, k, *, b, h, scale, causal, window=0, key_mask=None, mutation=0):
    """L x S softmax weights of one (batch, query head)."""
    qb, kb = _bits(q), _bits(k)
    B, Hq, Hkv, L, S, D = _shape(qb, kb)
    km = _mask(key_mask)
    W = np.empty((L, S), dtype=np.float64)
    code = MUTATIONS[mutation] if isinstance(mutation, str) else int(mutation)
    rc = _load().oracle_softmax_weights(_ptr(qb), _ptr(kb), _ptr(W), B, Hq, Hkv, L, S, D,
                                        float(scale), int(bool(causal)), int(window), _ptr(km),
                                        int(b), int(h), code)
    if rc:
        raise ValueError(f"oracle_softmax_weights rejected its arguments (code {rc})")
    return W


def allowed(L, S, i, j, *, causal, window=0, key_mask_row=None) -> bool:
    km = _mask(key_mask_row)
    return bool(_load().oracle_allowed(L, S, i, j, int(bool(causal)), int(window), _ptr(km)))


def visibility(L, S, *, causal, window=0, key_mask_row=None) -> np.ndarray:
    """L x S boolean matrix of allowed (row, key) pairs."""
    return np.array([[allowed(L, S, i, j, causal=causal, window=window, key_mask_row=key_mask_row)
                      for j in range(S)] for i in range(L)], dtype=bool)


def count_pairs(B, Hq, L, S, *, causal, window=0, key_mask=None) -> int:
    km = _mask(key_mask)
    return int(_load().oracle_count_pairs(B, Hq, L, S, int(bool(causal)), int(window), _ptr(km)))
