"""fp64 CPU oracle for ring-scheduled blockwise softmax attention.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this package.  The product library neither
imports nor links it, and it shares no code with the CUDA path.

What it computes is the plain definition of softmax attention and of the
log-sum-exp merge from "上下文并行与 Ring Attention" (hs-black.github.io),
section 分块注意力: see oracle.c for the formulas and layout.py for the token
layouts (sections Ring Attention, Zig-zag, Striped, 重排 token 的代价).

Inputs are numpy arrays; they are upcast to float64 before the C code sees
them, so bf16/fp32 device inputs enter the oracle exactly.
"""
import ctypes
import os

import numpy as np

from . import layout  # noqa: F401  (re-exported)
from .build import build as _build

_lib = None
_I64P = ctypes.POINTER(ctypes.c_int64)
_F64P = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build())
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [_F64P, _F64P, _F64P, _I64P, _I64P] + \
            [ctypes.c_int64] * 6 + [ctypes.c_int, ctypes.c_double, _F64P, _F64P, ctypes.c_int]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = [_F64P, _I64P, ctypes.c_int64, _F64P, _F64P, _I64P] + \
            [ctypes.c_int64] * 5 + [ctypes.c_int, ctypes.c_double, _F64P, _F64P, ctypes.c_int]
        lib.oracle_lse_merge.restype = None
        lib.oracle_lse_merge.argtypes = [ctypes.c_int64, ctypes.c_int64] + [_F64P] * 6
        _lib = lib
    return _lib


def default_threads():
    return len(os.sched_getaffinity(0))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def attention(q, k, v, causal, scale, pos_q=None, pos_k=None, nthreads=None):
    """Softmax attention by definition.

    q [b, sq, hq, d]; k, v [b, sk, hkv, d]; pos_q [sq], pos_k [sk] original
    positions (identity when None).  Returns (o [b, sq, hq, d], lse [b, hq, sq])
    in float64; rows with no visible key get o = 0, lse = -inf.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, sq, hq, d = q.shape
    bk, sk, hkv, dk = k.shape
    if bk != b or dk != d or v.shape != k.shape:
        raise ValueError("shape mismatch")
    pq = None if pos_q is None else np.ascontiguousarray(pos_q, dtype=np.int64)
    pk = None if pos_k is None else np.ascontiguousarray(pos_k, dtype=np.int64)
    if pq is not None and pq.shape != (sq,):
        raise ValueError("pos_q shape")
    if pk is not None and pk.shape != (sk,):
        raise ValueError("pos_k shape")
    o = np.empty((b, sq, hq, d), np.float64)
    lse = np.empty((b, hq, sq), np.float64)
    rc = _load().oracle_attention(_ptr(q, _F64P), _ptr(k, _F64P), _ptr(v, _F64P), _ptr(pq, _I64P),
                                  _ptr(pk, _I64P), b, sq, sk, hq, hkv, d, int(bool(causal)),
                                  float(scale), _ptr(o, _F64P), _ptr(lse, _F64P),
                                  nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")
    return o, lse


def attention_rows(q_sel, sel, k, v, causal, scale, hq, pos_k=None, nthreads=None):
    """Attention for selected query rows only.

    q_sel [n, d]; sel [n, 3] integer (batch, q head, original query position);
    k, v [b, sk, hkv, d].  Returns (o [n, d], lse [n]) in float64.
    """
    q_sel = _f64(q_sel)
    sel = np.ascontiguousarray(sel, dtype=np.int64)
    k, v = _f64(k), _f64(v)
    b, sk, hkv, d = k.shape
    n = sel.shape[0]
    pk = None if pos_k is None else np.ascontiguousarray(pos_k, dtype=np.int64)
    o = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_attention_rows(_ptr(q_sel, _F64P), _ptr(sel, _I64P), n, _ptr(k, _F64P),
                                       _ptr(v, _F64P), _ptr(pk, _I64P), b, sk, hq, hkv, d,
                                       int(bool(causal)), float(scale), _ptr(o, _F64P),
                                       _ptr(lse, _F64P), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_rows rejected its arguments")
    return o, lse


def lse_merge(o1, lse1, o2, lse2):
    """Stable two-way merge of partials; o* [..., d], lse* [...] (same leading shape)."""
    o1, o2, lse1, lse2 = _f64(o1), _f64(o2), _f64(lse1), _f64(lse2)
    d = o1.shape[-1]
    n = lse1.size
    if o1.size != n * d or o2.shape != o1.shape or lse2.shape != lse1.shape:
        raise ValueError("shape mismatch")
    o = np.empty_like(o1)
    lse = np.empty_like(lse1)
    _load().oracle_lse_merge(n, d, _ptr(o1, _F64P), _ptr(lse1, _F64P), _ptr(o2, _F64P),
                             _ptr(lse2, _F64P), _ptr(o, _F64P), _ptr(lse, _F64P))
    return o, lse


def ring_attention(q, k, v, layout_name, n_ranks, causal, scale, nthreads=None):
    """Reference result of ring attention on original-order tensors.

    The method reaches full softmax attention exactly (same page, 分块注意力:
    the split result equals one-shot softmax), so this is the plain definition
    over the whole sequence; the layout and N only permute tokens.  Returns
    (o [b, S, hq, d], lse [b, hq, S]) in ORIGINAL token order.
    """
    layout.tokens_per_rank(layout_name, n_ranks, q.shape[1])
    return attention(q, k, v, causal, scale, nthreads=nthreads)
