"""ctypes binding of libtfa.so -- argument marshalling only.

Every entry point of ``include/tfa.h`` is exposed under the same name and
takes the same arguments (pointers as Python ints).  ``prefill`` is the
convenience wrapper a PyTorch user calls: it checks dtypes/devices, allocates
the output with PyTorch and passes raw pointers and the current stream to
``tfa_prefill``.  There is no fallback: if the library is missing or the call
fails, it raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtfa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "tfa.h")

TFA_OK = 0
TFA_ERR_NULL = 1
TFA_ERR_HEADS = 2
TFA_ERR_SHORT_QUERY = 3
TFA_ERR_SHAPE = 4
TFA_ERR_HEAD_DIM = 5
TFA_ERR_WINDOW = 6
TFA_ERR_ALIGN = 7
TFA_ERR_CUDA = 8
TFA_ERR_TIMEOUT = 9
TFA_ERR_SCALE = 10
TFA_ERR_FLAGS = 11
TFA_ERR_CAPTURE = 12
TFA_ERR_SOFTCAP = 13
TFA_ERR_SEQLENS = 14
TFA_ERR_RING = 15
MAX_VARLEN_SEQS = 1024

TFA_DEBUG_NO_TILE_SKIP = 1
TFA_DEBUG_MASK_ALL = 2
TFA_DEBUG_SYNC = 4
TFA_DEBUG_NO_SPLIT = 8
TFA_DEBUG_FORCE_SPLIT = 16
TFA_DEBUG_SHORT_WAITS = 32

MIN_QUERY_ROWS = 9
MAX_DECODE_ROWS = 8
BLOCK_Q = 128
BLOCK_K = 128

_lock = threading.Lock()
_lib = None


class TfaError(RuntimeError):
    def __init__(self, code: int, where: str = "tfa_prefill"):
        self.code = code
        detail = f" [{last_error()}]" if code in (TFA_ERR_CUDA, TFA_ERR_CAPTURE) else ""
        super().__init__(f"{where} failed with status {code}: {status_string(code)}{detail}")


def lib():
    """Load libtfa.so; raise if it has not been built (no fallback path exists)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m sliding_window_gqa_tfa_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, u32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_float
            common = [P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, P, P]
            L.tfa_prefill.argtypes = common
            L.tfa_prefill.restype = i32
            L.tfa_prefill_debug.argtypes = common + [u32]
            L.tfa_prefill_debug.restype = i32
            L.tfa_prefill_host.argtypes = common
            L.tfa_prefill_host.restype = i32
            L.tfa_prefill_noalloc.argtypes = common
            L.tfa_prefill_noalloc.restype = i32
            L.tfa_decode.argtypes = common
            L.tfa_decode.restype = i32
            L.tfa_attention_ex.argtypes = common[:14] + [f32, P, P]
            L.tfa_attention_ex.restype = i32
            L.tfa_prefill_backward.argtypes = [P] * 7 + [i32] * 6 + [f32, i32, i32, P, P]
            L.tfa_prefill_backward.restype = i32
            L.tfa_prefill_lse.argtypes = [P] * 5 + [i32] * 6 + [f32, i32, i32, P, P]
            L.tfa_prefill_lse.restype = i32
            L.tfa_prefill_backward_saved.argtypes = [P] * 9 + [i32] * 6 + [f32, i32, i32, P, P]
            L.tfa_prefill_backward_saved.restype = i32
            L.tfa_prefill_ring.argtypes = [P, P, P, P] + [i32] * 7 + [f32, i32, f32, P, P]
            L.tfa_prefill_ring.restype = i32
            L.tfa_prefill_varlen.argtypes = [P] * 6 + [i32] * 7 + [f32, i32, i32, f32, P, P]
            L.tfa_prefill_varlen.restype = i32
            L.tfa_check_status.argtypes = [P]
            L.tfa_check_status.restype = i32
            L.tfa_last_error.argtypes = []
            L.tfa_last_error.restype = ctypes.c_char_p
            L.tfa_status_string.argtypes = [i32]
            L.tfa_status_string.restype = ctypes.c_char_p
            L.tfa_plan_qtile.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(i32),
                                         ctypes.POINTER(i32), P, i32]
            L.tfa_plan_qtile.restype = i32
            L.tfa_plan_ktile.argtypes = [i32] * 5 + [ctypes.POINTER(i32), ctypes.POINTER(i32)]
            L.tfa_plan_ktile.restype = i32
            L.tfa_plan_pieces.argtypes = [i32] * 9 + [P, i32, ctypes.POINTER(i32),
                                                      ctypes.POINTER(ctypes.c_longlong)]
            L.tfa_plan_pieces.restype = i32
            _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Names of the functions include/tfa.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char \*)\s*(tfa_\w+)\s*\(", text, re.M)))


def last_error() -> str:
    return lib().tfa_last_error().decode()


def status_string(code: int) -> str:
    return lib().tfa_status_string(int(code)).decode()


# ----------------------------------------------------------- raw entry points
def tfa_attention_ex(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, softcap,
                     sinks, stream) -> int:
    return lib().tfa_attention_ex(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                                  softcap, sinks, stream)


def tfa_prefill_ring(q, k, v, o, B, Hq, Hkv, L, S, ring_rows, D, scale, window, softcap, sinks,
                     stream) -> int:
    return lib().tfa_prefill_ring(q, k, v, o, B, Hq, Hkv, L, S, ring_rows, D, scale, window,
                                  softcap, sinks, stream)


def tfa_prefill_varlen(q, k, v, o, cu_q, cu_k, B, Hq, Hkv, total_q, total_k, max_seqlen_q, D,
                       scale, causal, window, softcap, sinks, stream) -> int:
    return lib().tfa_prefill_varlen(q, k, v, o, cu_q, cu_k, B, Hq, Hkv, total_q, total_k,
                                    max_seqlen_q, D, scale, causal, window, softcap, sinks, stream)


def tfa_prefill(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, stream) -> int:
    return lib().tfa_prefill(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                             stream)


def tfa_prefill_debug(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, stream,
                      flags) -> int:
    return lib().tfa_prefill_debug(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window,
                                   key_mask, stream, flags)


def tfa_prefill_host(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                     stream) -> int:
    return lib().tfa_prefill_host(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window,
                                  key_mask, stream)


def tfa_decode(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, stream) -> int:
    return lib().tfa_decode(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                            stream)


def tfa_prefill_noalloc(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                        stream) -> int:
    return lib().tfa_prefill_noalloc(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window,
                                     key_mask, stream)


def tfa_check_status(stream) -> int:
    return lib().tfa_check_status(stream)


def tfa_plan_qtile(L, S, causal, window, has_key_mask, qtile):
    """Returns (status, kt_lo, kt_hi, needs_mask list)."""
    lo, hi = ctypes.c_int(0), ctypes.c_int(0)
    buf = (ctypes.c_ubyte * (S // BLOCK_K + 2))()
    rc = lib().tfa_plan_qtile(L, S, int(causal), window, int(has_key_mask), qtile,
                              ctypes.byref(lo), ctypes.byref(hi),
                              ctypes.cast(buf, ctypes.c_void_p), len(buf))
    if rc:
        return rc, None, None, None
    return rc, lo.value, hi.value, [bool(buf[i]) for i in range(hi.value - lo.value + 1)]


def tfa_plan_ktile(L, S, causal, window, ktile):
    """(status, first query tile, last query tile) that see key tile `ktile`."""
    lo, hi = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib().tfa_plan_ktile(L, S, int(bool(causal)), window, ktile, ctypes.byref(lo), ctypes.byref(hi))
    return rc, lo.value, hi.value


def tfa_plan_pieces(B, Hq, L, S, causal, window, grid, split, cta, max_pieces=4096):
    """Returns (status, total_steps, pieces) with pieces as tuples of 10 ints."""
    buf = (ctypes.c_int * (10 * max_pieces))()
    n = ctypes.c_int(0)
    w = ctypes.c_longlong(0)
    rc = lib().tfa_plan_pieces(B, Hq, L, S, int(causal), window, grid, int(split), cta,
                               ctypes.cast(buf, ctypes.c_void_p), max_pieces, ctypes.byref(n),
                               ctypes.byref(w))
    if rc:
        return rc, None, None
    return rc, w.value, [tuple(buf[10 * i:10 * i + 10]) for i in range(n.value)]


# ---------------------------------------------------------- torch wrapper
def _stream_handle(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(t, name, dtype, ndim):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill(q, k, v, *, scale=None, causal=True, window=0, key_mask=None, out=None, stream=None,
            debug_flags=0, softcap=0.0, sinks=None):
    """Attention output [B,Hq,L,D] bf16 for bf16 q [B,Hq,L,D], k/v [B,Hkv,S,D] on one GPU.

    L >= 9 goes to tfa_prefill, 1 <= L <= 8 to tfa_decode; a softcap > 0 or
    sinks (fp32 [Hq] on the device) go to tfa_attention_ex.  key_mask: optional
    fp32 [B,S] (1 keep / 0 drop).  Raises TfaError on a nonzero status."""
    import torch

    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    B, Hq, L, D = q.shape
    Bk, Hkv, S, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must have the same shape")
    if Bk != B or Dk != D:
        raise ValueError("q and k disagree on batch or head dimension")
    if key_mask is not None:
        _check(key_mask, "key_mask", torch.float32, 2)
        if tuple(key_mask.shape) != (B, S):
            raise ValueError("key_mask must be [B, S]")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", torch.bfloat16, 4)
        if tuple(out.shape) != tuple(q.shape):
            raise ValueError("out must have q's shape")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    args = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, Hq, Hkv, L, S, D,
            float(scale), int(bool(causal)), int(window),
            ctypes.c_void_p(key_mask.data_ptr()) if key_mask is not None else None,
            _stream_handle(stream))
    if softcap or sinks is not None:
        if debug_flags:
            raise ValueError("debug flags apply to tfa_prefill_debug only")
        if sinks is not None:
            _check(sinks, "sinks", torch.float32, 1)
            if sinks.shape[0] != Hq:
                raise ValueError("sinks must hold one logit per query head")
        rc = tfa_attention_ex(*args[:14], float(softcap),
                              ctypes.c_void_p(sinks.data_ptr()) if sinks is not None else None,
                              args[14])
        if rc != TFA_OK:
            raise TfaError(rc, "tfa_attention_ex")
        return out
    if L <= MAX_DECODE_ROWS:
        if debug_flags:
            raise ValueError("debug flags apply to the prefill path only (L >= 9)")
        rc = tfa_decode(*args)
        if rc != TFA_OK:
            raise TfaError(rc, "tfa_decode")
        return out
    rc = tfa_prefill_debug(*args, debug_flags) if debug_flags else tfa_prefill(*args)
    if rc != TFA_OK:
        raise TfaError(rc)
    return out


def tfa_prefill_backward(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, D, scale, causal, window,
                         key_mask, stream) -> int:
    return lib().tfa_prefill_backward(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, D, scale, causal,
                                      window, key_mask, stream)


def prefill_lse(q, k, v, *, scale=None, causal=True, window=0, key_mask=None, out=None, lse=None,
                stream=None):
    """(o, lse): the forward of any L >= 1 and each row's base-2 log-sum-exp of
    its scaled scores, fp32 [B,Hq,L] (+inf for a row with no allowed key)."""
    import torch

    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 4)
    B, Hq, L, D = q.shape
    Bk, Hkv, S, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D:
        raise ValueError("q, k and v disagree")
    if key_mask is not None:
        _check(key_mask, "key_mask", torch.float32, 2)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    rc = lib().tfa_prefill_lse(*(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, out, lse)),
                               B, Hq, Hkv, L, S, D, float(scale), int(bool(causal)), int(window),
                               _ptr_or_none(key_mask), _stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_prefill_lse")
    return out, lse


def backward(q, k, v, dout, *, scale=None, causal=True, window=0, key_mask=None, out=None,
             saved=None, stream=None):
    """(dq, dk, dv) bf16 of the attention core for the upstream gradient dout
    [B,Hq,L,D]: recompute-based (the forward is re-run inside), or, given
    saved=(o, lse) from prefill_lse on the same inputs, from those."""
    import torch

    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _check(t, n, torch.bfloat16, 4)
    B, Hq, L, D = q.shape
    Bk, Hkv, S, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or tuple(dout.shape) != tuple(q.shape) or Bk != B or Dk != D:
        raise ValueError("q, k, v and dout disagree")
    if key_mask is not None:
        _check(key_mask, "key_mask", torch.float32, 2)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = out
    for t, ref, n in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _check(t, n, torch.bfloat16, 4)
        if tuple(t.shape) != tuple(ref.shape):
            raise ValueError(f"{n} has the wrong shape")
    if saved is not None:
        o, lse = saved
        _check(o, "o", torch.bfloat16, 4)
        _check(lse, "lse", torch.float32, 3)
        if tuple(o.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, L):
            raise ValueError("saved (o, lse) have the wrong shape")
        rc = lib().tfa_prefill_backward_saved(
            *(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, o, lse, dout, dq, dk, dv)),
            B, Hq, Hkv, L, S, D, float(scale), int(bool(causal)), int(window), _ptr_or_none(key_mask),
            _stream_handle(stream))
        if rc != TFA_OK:
            raise TfaError(rc, "tfa_prefill_backward_saved")
        return dq, dk, dv
    rc = tfa_prefill_backward(*(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, dout, dq, dk, dv)),
                              B, Hq, Hkv, L, S, D, float(scale), int(bool(causal)), int(window),
                              _ptr_or_none(key_mask), _stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_prefill_backward")
    return dq, dk, dv


def _ptr_or_none(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def prefill_ring(q, k_ring, v_ring, *, S, window, scale=None, softcap=0.0, sinks=None, out=None,
                 stream=None):
    """Attention over a rotating K/V cache: k_ring/v_ring [B,Hkv,R,D] bf16 hold the
    last R positions, position j in row j mod R; q [B,Hq,L,D] are the newest L
    positions of S.  Causal with a window (R >= window - 1 + L, R a multiple of 64)."""
    import torch

    _check(q, "q", torch.bfloat16, 4)
    _check(k_ring, "k_ring", torch.bfloat16, 4)
    _check(v_ring, "v_ring", torch.bfloat16, 4)
    B, Hq, L, D = q.shape
    Bk, Hkv, R, Dk = k_ring.shape
    if tuple(v_ring.shape) != tuple(k_ring.shape) or Bk != B or Dk != D:
        raise ValueError("q, k_ring and v_ring disagree")
    if sinks is not None:
        _check(sinks, "sinks", torch.float32, 1)
    out = torch.empty_like(q) if out is None else out
    _check(out, "out", torch.bfloat16, 4)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = tfa_prefill_ring(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_ring.data_ptr()),
                          ctypes.c_void_p(v_ring.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                          B, Hq, Hkv, L, int(S), R, D, float(scale), int(window), float(softcap),
                          _ptr_or_none(sinks), _stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_prefill_ring")
    return out


def prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, *, max_seqlen_q, scale=None, causal=True,
                   window=0, softcap=0.0, sinks=None, out=None, stream=None):
    """Packed variable-length attention: q [Tq,Hq,D], k/v [Tk,Hkv,D] bf16, int32 device
    prefix sums cu_seqlens_* [B+1].  Returns out [Tq,Hq,D]."""
    import torch

    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    Tq, Hq, D = q.shape
    Tk, Hkv, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Dk != D:
        raise ValueError("q, k and v disagree")
    B = cu_seqlens_q.shape[0] - 1
    if cu_seqlens_k.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    if sinks is not None:
        _check(sinks, "sinks", torch.float32, 1)
    out = torch.empty_like(q) if out is None else out
    _check(out, "out", torch.bfloat16, 3)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = tfa_prefill_varlen(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                            ctypes.c_void_p(cu_seqlens_q.data_ptr()),
                            ctypes.c_void_p(cu_seqlens_k.data_ptr()), B, Hq, Hkv, Tq, Tk,
                            int(max_seqlen_q), D, float(scale), int(bool(causal)), int(window),
                            float(softcap), _ptr_or_none(sinks), _stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_prefill_varlen")
    return out


def check_status(stream=None) -> None:
    """Synchronize `stream` and raise TfaError if a kernel recorded a timed-out wait."""
    rc = tfa_check_status(_stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_check_status")


def prefill_host(q, k, v, *, scale=None, causal=True, window=0, key_mask=None, out=None,
                 stream=None):
    """The same operation on CPU tensors (pinned or pageable) through tfa_prefill_host."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
    B, Hq, L, D = q.shape
    _, Hkv, S, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    km = None
    if key_mask is not None:
        if key_mask.dtype != torch.float32 or key_mask.is_cuda or not key_mask.is_contiguous():
            raise ValueError("key_mask must be a contiguous fp32 CPU tensor")
        km = ctypes.c_void_p(key_mask.data_ptr())
    rc = tfa_prefill_host(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                          ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                          B, Hq, Hkv, L, S, D, float(scale), int(bool(causal)), int(window), km,
                          _stream_handle(stream))
    if rc != TFA_OK:
        raise TfaError(rc, "tfa_prefill_host")
    return out
