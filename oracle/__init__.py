"""fp64 CPU oracle for ring-scheduled blockwise softmax attention.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this package.  The product library neither
imports nor links it, and it shares no code with the CUDA path.

What it computes is the plain definition of softmax attention and of the
log-sum-exp merge from "上下文并行与 Ring Attention" (hs-black.github.io),
section 分块注意力, and of its gradients (the same section's paragraph on the
backward pass): see oracle.c for the formulas and layout.py for the token
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
        _bwd_sigs(lib)
        lib.oracle_attention_bwd_doc.restype = ctypes.c_int
        lib.oracle_attention_bwd_doc.argtypes = [_F64P] * 4 + [_I64P] * 2 + [ctypes.c_int64] * 6 + \
            [ctypes.c_int, _I64P, ctypes.c_int64, ctypes.c_double] + [_F64P] * 3 + [ctypes.c_int]
        lib.oracle_attention_doc.restype = ctypes.c_int
        lib.oracle_attention_doc.argtypes = [_F64P, _F64P, _F64P, _I64P, _I64P] + [ctypes.c_int64] * 6 + \
            [ctypes.c_int, _I64P, ctypes.c_int64, ctypes.c_double, _F64P, _F64P, ctypes.c_int]
        lib.oracle_attention_rows_doc.restype = ctypes.c_int
        lib.oracle_attention_rows_doc.argtypes = [_F64P, _I64P, ctypes.c_int64, _F64P, _F64P, _I64P] + \
            [ctypes.c_int64] * 5 + [ctypes.c_int, _I64P, ctypes.c_int64, ctypes.c_double, _F64P, _F64P, ctypes.c_int]
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


def _bwd_sigs(lib):
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [_F64P] * 4 + [_I64P] * 2 + [ctypes.c_int64] * 6 + \
        [ctypes.c_int, ctypes.c_double] + [_F64P] * 7 + [ctypes.c_int]
    lib.oracle_attention_bwd_sel.restype = ctypes.c_int
    lib.oracle_attention_bwd_sel.argtypes = [_F64P] * 4 + [_I64P] * 2 + [ctypes.c_int64] * 6 + \
        [ctypes.c_int, ctypes.c_double, _I64P, ctypes.c_int64, _F64P, _I64P, ctypes.c_int64, _F64P, _F64P,
         ctypes.c_int]


def _opt_pos(pos, n, what):
    if pos is None:
        return None
    a = np.ascontiguousarray(pos, dtype=np.int64)
    if a.shape != (n,):
        raise ValueError(what + " shape")
    return a


def attention_bwd(q, k, v, do, causal, scale, pos_q=None, pos_k=None, lse=None, delta=None, nthreads=None):
    """Gradients of softmax attention (section 分块注意力, backward paragraph).

    q, do [b, sq, hq, d]; k, v [b, sk, hkv, d].  With lse = delta = None the
    row statistics (lse, D = do . o) come from the definition over these keys;
    otherwise lse, delta [b, hq, sq] are the rows' GLOBAL statistics and the
    result is this key block's share of the gradients.  Returns
    (dq, dk, dv, lse, delta) in float64.
    """
    lib = _load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    b, sq, hq, d = q.shape
    bk, sk, hkv, dk_ = k.shape
    if bk != b or dk_ != d or v.shape != k.shape or do.shape != q.shape:
        raise ValueError("shape mismatch")
    if (lse is None) != (delta is None):
        raise ValueError("give both lse and delta, or neither")
    lse_in = None if lse is None else _f64(lse).reshape(b, hq, sq)
    delta_in = None if delta is None else _f64(delta).reshape(b, hq, sq)
    pq, pk = _opt_pos(pos_q, sq, "pos_q"), _opt_pos(pos_k, sk, "pos_k")
    dq = np.empty_like(q)
    dkk = np.empty_like(k)
    dv = np.empty_like(v)
    lse_out = np.empty((b, hq, sq), np.float64)
    delta_out = np.empty((b, hq, sq), np.float64)
    rc = lib.oracle_attention_bwd(_ptr(q, _F64P), _ptr(k, _F64P), _ptr(v, _F64P), _ptr(do, _F64P),
                                  _ptr(pq, _I64P), _ptr(pk, _I64P), b, sq, sk, hq, hkv, d, int(bool(causal)),
                                  float(scale), _ptr(lse_in, _F64P), _ptr(delta_in, _F64P), _ptr(dq, _F64P),
                                  _ptr(dkk, _F64P), _ptr(dv, _F64P), _ptr(lse_out, _F64P),
                                  _ptr(delta_out, _F64P), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_bwd rejected its arguments")
    return dq, dkk, dv, lse_out, delta_out


def attention_bwd_sel(q, k, v, do, causal, scale, sel_q, sel_k, pos_q=None, pos_k=None, nthreads=None):
    """Gradients at selected rows: sel_q [n, 3] = (batch, q head, query index) gives
    dq [n, d]; sel_k [m, 3] = (batch, kv head, key index) gives dk, dv [m, d]."""
    lib = _load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    b, sq, hq, d = q.shape
    _, sk, hkv, _ = k.shape
    sq_sel = np.ascontiguousarray(np.asarray(sel_q, dtype=np.int64).reshape(-1, 3))
    sk_sel = np.ascontiguousarray(np.asarray(sel_k, dtype=np.int64).reshape(-1, 3))
    pq, pk = _opt_pos(pos_q, sq, "pos_q"), _opt_pos(pos_k, sk, "pos_k")
    dq = np.empty((sq_sel.shape[0], d), np.float64)
    dkk = np.empty((sk_sel.shape[0], d), np.float64)
    dv = np.empty((sk_sel.shape[0], d), np.float64)
    rc = lib.oracle_attention_bwd_sel(_ptr(q, _F64P), _ptr(k, _F64P), _ptr(v, _F64P), _ptr(do, _F64P),
                                      _ptr(pq, _I64P), _ptr(pk, _I64P), b, sq, sk, hq, hkv, d,
                                      int(bool(causal)), float(scale), _ptr(sq_sel, _I64P), sq_sel.shape[0],
                                      _ptr(dq, _F64P), _ptr(sk_sel, _I64P), sk_sel.shape[0], _ptr(dkk, _F64P),
                                      _ptr(dv, _F64P), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_bwd_sel rejected its arguments")
    return dq, dkk, dv


def ring_attention_bwd(q, k, v, do, layout_name, n_ranks, causal, scale, nthreads=None):
    """Reference gradients of ring attention on original-order tensors.

    The ring reaches the plain definition's gradients exactly (section 分块注意力,
    backward paragraph: each block's share uses the global statistics), so this
    is the definition over the whole sequence; layout and N only permute tokens.
    Returns (dq, dk, dv) in ORIGINAL token order.
    """
    layout.tokens_per_rank(layout_name, n_ranks, q.shape[1])
    dq, dk, dv, _, _ = attention_bwd(q, k, v, do, causal, scale, nthreads=nthreads)
    return dq, dk, dv


def ring_attention_bwd_steps(q, k, v, do, layout_name, n_ranks, causal, scale, nthreads=None):
    """The ring's backward walked step by step, in the page's order.

    The forward's global (lse, D) of every query row come first.  Then at step r
    rank i holds the K/V block of rank (i - r) mod N together with that block's
    travelling dK, dV accumulators (section Ring Attention); it adds the block's
    share to its local dQ and to the travelling dK, dV.  After N steps every
    accumulator holds the full sum.  Returns (dq, dk, dv) in ORIGINAL token order.
    """
    S = q.shape[1]
    layout.tokens_per_rank(layout_name, n_ranks, S)
    o, lse = attention(q, k, v, causal, scale, nthreads=nthreads)
    delta = np.einsum("bshd,bshd->bhs", _f64(do), o)
    pos = [np.asarray(layout.rank_positions(layout_name, n_ranks, S, i), dtype=np.int64) for i in range(n_ranks)]
    dq = np.zeros(_f64(q).shape)
    dk = np.zeros(_f64(k).shape)
    dv = np.zeros(_f64(v).shape)
    for r in range(n_ranks):
        for i in range(n_ranks):
            src = (i - r) % n_ranks
            pi, pj = pos[i], pos[src]
            gq, gk, gv, _, _ = attention_bwd(q[:, pi], k[:, pj], v[:, pj], do[:, pi], causal, scale,
                                             pos_q=pi, pos_k=pj, lse=lse[:, :, pi], delta=delta[:, :, pi],
                                             nthreads=nthreads)
            dq[:, pi] += gq
            dk[:, pj] += gk
            dv[:, pj] += gv
    return dq, dk, dv


def _docs(doc_starts):
    d = np.ascontiguousarray(doc_starts, dtype=np.int64)
    if d.ndim != 1 or d.size < 1 or d[0] != 0 or np.any(np.diff(d) <= 0):
        raise ValueError("doc_starts must be strictly increasing and start at 0")
    return d


def attention_doc(q, k, v, causal, scale, doc_starts, pos_q=None, pos_k=None, nthreads=None):
    """Attention with a document mask (section All-Gather 式 CP: documents packed
    into one sequence do not see each other).  doc_starts: sorted first positions
    of the documents, starting with 0.  Otherwise as attention()."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, sq, hq, d = q.shape
    bk, sk, hkv, dk = k.shape
    if bk != b or dk != d or v.shape != k.shape:
        raise ValueError("shape mismatch")
    pq, pk = _opt_pos(pos_q, sq, "pos_q"), _opt_pos(pos_k, sk, "pos_k")
    docs = _docs(doc_starts)
    o = np.empty((b, sq, hq, d), np.float64)
    lse = np.empty((b, hq, sq), np.float64)
    rc = _load().oracle_attention_doc(_ptr(q, _F64P), _ptr(k, _F64P), _ptr(v, _F64P), _ptr(pq, _I64P),
                                      _ptr(pk, _I64P), b, sq, sk, hq, hkv, d, int(bool(causal)), _ptr(docs, _I64P),
                                      docs.size, float(scale), _ptr(o, _F64P), _ptr(lse, _F64P),
                                      nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_doc rejected its arguments")
    return o, lse


def attention_rows_doc(q_sel, sel, k, v, causal, scale, hq, doc_starts, pos_k=None, nthreads=None):
    """attention_rows() with the document mask."""
    q_sel = _f64(q_sel)
    sel = np.ascontiguousarray(sel, dtype=np.int64)
    k, v = _f64(k), _f64(v)
    b, sk, hkv, d = k.shape
    n = sel.shape[0]
    pk = _opt_pos(pos_k, sk, "pos_k")
    docs = _docs(doc_starts)
    o = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_attention_rows_doc(_ptr(q_sel, _F64P), _ptr(sel, _I64P), n, _ptr(k, _F64P),
                                           _ptr(v, _F64P), _ptr(pk, _I64P), b, sk, hq, hkv, d, int(bool(causal)),
                                           _ptr(docs, _I64P), docs.size, float(scale), _ptr(o, _F64P),
                                           _ptr(lse, _F64P), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_rows_doc rejected its arguments")
    return o, lse


def allgather_attention(q, k, v, layout_name, n_ranks, causal, scale, doc_starts, nthreads=None):
    """Reference result of All-Gather context parallelism (section All-Gather 式 CP)
    on original-order tensors: every rank sees the whole K/V, so the result is the
    plain definition with the document mask over the whole sequence.  Returns
    (o, lse) in ORIGINAL token order."""
    layout.tokens_per_rank(layout_name, n_ranks, q.shape[1])
    return attention_doc(q, k, v, causal, scale, doc_starts, nthreads=nthreads)


def allgather_attention_steps(q, k, v, layout_name, n_ranks, causal, scale, doc_starts, nthreads=None):
    """The All-Gather schedule written out: K and V gathered into one original-order
    copy, then each rank's queries (its layout positions) attend to all of it."""
    S = q.shape[1]
    layout.tokens_per_rank(layout_name, n_ranks, S)
    q64 = _f64(q)
    o = np.zeros(q64.shape)
    lse = np.zeros((q64.shape[0], q64.shape[2], S))
    for i in range(n_ranks):
        pos = np.asarray(layout.rank_positions(layout_name, n_ranks, S, i), dtype=np.int64)
        oi, li = attention_doc(q64[:, pos], k, v, causal, scale, doc_starts, pos_q=pos, nthreads=nthreads)
        o[:, pos] = oi
        lse[:, :, pos] = li
    return o, lse


def ulysses_all_to_all(x, n_ranks, inverse=False):
    """The Ulysses exchange written out (section DeepSpeed-Ulysses): block (s_i, h_j)
    moves from rank i to rank j.  Forward: x [b, S, H, d] with rank i holding tokens
    [i S/P, (i+1) S/P) -> [P, b, S, H/P, d] (rank j: all tokens, heads
    [j H/P, (j+1) H/P)).  Inverse: the reverse.  A pure index map in numpy."""
    P = n_ranks
    if not inverse:
        b, S, H, d = x.shape
        c, hp = S // P, H // P
        out = np.empty((P, b, S, hp, d), dtype=x.dtype)
        for i in range(P):          # source rank: sequence shard i
            for j in range(P):      # destination rank: head group j
                out[j, :, i * c:(i + 1) * c] = x[:, i * c:(i + 1) * c, j * hp:(j + 1) * hp]
        return out
    P_, b, S, hp, d = x.shape
    c = S // P
    out = np.empty((b, S, hp * P, d), dtype=x.dtype)
    for j in range(P):
        for i in range(P):
            out[:, i * c:(i + 1) * c, j * hp:(j + 1) * hp] = x[j, :, i * c:(i + 1) * c]
    return out


def ulysses_attention(q, k, v, n_ranks, causal, scale, nthreads=None):
    """Reference result of Ulysses attention: heads are independent, so the exchange
    around per-head-group attention reproduces plain attention exactly."""
    if q.shape[2] % n_ranks or k.shape[2] % n_ranks or q.shape[1] % n_ranks:
        raise ValueError("P must divide the heads and the sequence")
    return attention(q, k, v, causal, scale, nthreads=nthreads)


def ulysses_attention_steps(q, k, v, n_ranks, causal, scale, nthreads=None):
    """The four steps of the page: all-to-all of q, k, v, each rank's attention over
    its n_h/P heads and the whole sequence, all-to-all of o (and lse) back."""
    P = n_ranks
    qh, kh, vh = (ulysses_all_to_all(_f64(t), P) for t in (q, k, v))
    b, S, Hq, d = _f64(q).shape
    hp = Hq // P
    oh = np.empty_like(qh)
    lh = np.empty((P, b, hp, S))
    for j in range(P):
        oh[j], lh[j] = attention(qh[j], kh[j], vh[j], causal, scale, nthreads=nthreads)
    o = ulysses_all_to_all(oh, P, inverse=True)
    lse = np.concatenate([lh[j] for j in range(P)], axis=1)  # [b, Hq, S], head group j at j*hp
    return o, lse


def ulysses_attention_bwd(q, k, v, do, n_ranks, causal, scale, nthreads=None):
    """Reference gradients of Ulysses attention: the plain definition (heads are
    independent).  Returns (dq, dk, dv) in original order."""
    if q.shape[2] % n_ranks or k.shape[2] % n_ranks or q.shape[1] % n_ranks:
        raise ValueError("P must divide the heads and the sequence")
    dq, dk, dv, _, _ = attention_bwd(q, k, v, do, causal, scale, nthreads=nthreads)
    return dq, dk, dv


def ulysses_attention_bwd_steps(q, k, v, do, n_ranks, causal, scale, nthreads=None):
    """Exchange of q, k, v, dO; each rank's head-group gradients over the whole
    sequence; exchange of dq, dk, dv back."""
    P = n_ranks
    qh, kh, vh, doh = (ulysses_all_to_all(_f64(t), P) for t in (q, k, v, do))
    g = [attention_bwd(qh[j], kh[j], vh[j], doh[j], causal, scale, nthreads=nthreads)[:3] for j in range(P)]
    return tuple(ulysses_all_to_all(np.stack([g[j][n] for j in range(P)]), P, inverse=True) for n in range(3))


def _usp_positions(layout_name, n_ring, n_uly, S):
    """Original positions held by rank (g, u) before the USP exchange: ring group g
    holds the ring layout's block g, its Ulysses rank u the u-th contiguous slice."""
    c = layout.tokens_per_rank(layout_name, n_ring, S)
    if c % n_uly:
        raise ValueError("the ring block must split into n_uly slices")
    cs = c // n_uly
    blocks = [np.asarray(layout.rank_positions(layout_name, n_ring, S, g), dtype=np.int64) for g in range(n_ring)]
    return blocks, {(g, u): blocks[g][u * cs:(u + 1) * cs] for g in range(n_ring) for u in range(n_uly)}


def usp_exchange(x, layout_name, n_ring, n_uly):
    """The USP exchange written out ("DeepSpeed-Ulysses" page, section on USP: the
    Ulysses all-to-all inside each group of the ring).  x [b, S, H, d] in original
    order.  Rank (g, u) starts with its slice of group g's block (all heads); inside
    the group, rank (g, u') sends the head group u of its slice to rank (g, u).
    Returns a dict (g, u) -> [b, c, H/P, d]: group g's block in layout order, head
    group u.  A pure index map."""
    S, H = x.shape[1], x.shape[2]
    P = n_uly
    if H % P:
        raise ValueError("n_uly must divide the heads")
    hp = H // P
    _, held = _usp_positions(layout_name, n_ring, n_uly, S)
    out = {}
    for g in range(n_ring):
        for u in range(P):      # destination rank (g, u)
            parts = [x[:, held[(g, u2)], u * hp:(u + 1) * hp] for u2 in range(P)]   # from (g, u2), in u2 order
            out[(g, u)] = np.concatenate(parts, axis=1)
    return out


def usp_attention(q, k, v, layout_name, n_ring, n_uly, causal, scale, nthreads=None):
    """Reference result of USP: heads are independent and the ring reaches full
    attention, so the hybrid reproduces the plain definition exactly.  Original
    order in and out."""
    if q.shape[2] % n_uly or k.shape[2] % n_uly:
        raise ValueError("n_uly must divide the heads")
    _usp_positions(layout_name, n_ring, n_uly, q.shape[1])
    return attention(q, k, v, causal, scale, nthreads=nthreads)


def usp_attention_steps(q, k, v, layout_name, n_ring, n_uly, causal, scale, nthreads=None):
    """USP step by step: the exchange inside every group, then for every head group
    the ring over the N groups (at step r rank (g, u) holds the K/V block of rank
    ((g - r) mod N, u), attends its queries to it and merges the partial into its
    running (o, lse); section Ring Attention), then the exchange back.  Returns
    (o [b, S, Hq, d], lse [b, Hq, S]) in original order."""
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    b, S, Hq, d = q64.shape
    N, P = n_ring, n_uly
    hp = Hq // P
    blocks, held = _usp_positions(layout_name, N, P, S)
    qx, kx, vx = (usp_exchange(t, layout_name, N, P) for t in (q64, k64, v64))
    o = np.zeros(q64.shape)
    lse = np.zeros((b, Hq, S))
    for g in range(N):
        for u in range(P):
            acc_o = np.zeros((b, hp, blocks[g].size, d))
            acc_l = np.full((b, hp, blocks[g].size), -np.inf)
            for r in range(N):
                src = (g - r) % N
                ob, lb = attention(qx[(g, u)], kx[(src, u)], vx[(src, u)], causal, scale, pos_q=blocks[g],
                                   pos_k=blocks[src], nthreads=nthreads)
                acc_o, acc_l = lse_merge(acc_o, acc_l, ob.transpose(0, 2, 1, 3), lb)
            # exchange back: rank (g, u) returns slice u2 of its rows to rank (g, u2)
            cs = blocks[g].size // P
            for u2 in range(P):
                rows = slice(u2 * cs, (u2 + 1) * cs)
                o[:, held[(g, u2)], u * hp:(u + 1) * hp] = acc_o[:, :, rows].transpose(0, 2, 1, 3)
                lse[:, u * hp:(u + 1) * hp, held[(g, u2)]] = acc_l[:, :, rows]
    return o, lse


def usp_attention_bwd(q, k, v, do, layout_name, n_ring, n_uly, causal, scale, nthreads=None):
    """Reference gradients of USP: the plain definition's.  Original order."""
    if q.shape[2] % n_uly or k.shape[2] % n_uly:
        raise ValueError("n_uly must divide the heads")
    _usp_positions(layout_name, n_ring, n_uly, q.shape[1])
    dq, dk, dv, _, _ = attention_bwd(q, k, v, do, causal, scale, nthreads=nthreads)
    return dq, dk, dv


def usp_attention_bwd_steps(q, k, v, do, layout_name, n_ring, n_uly, causal, scale, nthreads=None):
    """USP backward step by step: the exchange of q, k, v, dO inside every group; per
    head group the global statistics of every row, then the ring over the groups
    with dK, dV travelling with their block (the block shares of section 分块注意力's
    backward paragraph); the exchange of dq, dk, dv back.  Original order."""
    q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(do)
    S, Hq, Hkv = q64.shape[1], q64.shape[2], k64.shape[2]
    N, P = n_ring, n_uly
    hp, hkp = Hq // P, Hkv // P
    blocks, held = _usp_positions(layout_name, N, P, S)
    qx, kx, vx, dox = (usp_exchange(t, layout_name, N, P) for t in (q64, k64, v64, do64))
    dq, dk, dv = np.zeros(q64.shape), np.zeros(k64.shape), np.zeros(v64.shape)
    for u in range(P):
        # global statistics of every row of head group u (the forward's lse, D = dO . o)
        stats = {}
        for g in range(N):
            kk = np.concatenate([kx[(j, u)] for j in range(N)], axis=1)
            vv = np.concatenate([vx[(j, u)] for j in range(N)], axis=1)
            pk = np.concatenate([blocks[j] for j in range(N)])
            og, lg = attention(qx[(g, u)], kk, vv, causal, scale, pos_q=blocks[g], pos_k=pk, nthreads=nthreads)
            stats[g] = (lg, np.einsum("bshd,bshd->bhs", dox[(g, u)], og))
        gq = {g: np.zeros(qx[(g, u)].shape) for g in range(N)}
        gk = {j: np.zeros(kx[(j, u)].shape) for j in range(N)}
        gv = {j: np.zeros(vx[(j, u)].shape) for j in range(N)}
        for r in range(N):
            for g in range(N):
                src = (g - r) % N
                a, bk, bv, _, _ = attention_bwd(qx[(g, u)], kx[(src, u)], vx[(src, u)], dox[(g, u)], causal, scale,
                                                pos_q=blocks[g], pos_k=blocks[src], lse=stats[g][0],
                                                delta=stats[g][1], nthreads=nthreads)
                gq[g] += a
                gk[src] += bk
                gv[src] += bv
        for g in range(N):
            cs = blocks[g].size // P
            for u2 in range(P):
                rows = slice(u2 * cs, (u2 + 1) * cs)
                dq[:, held[(g, u2)], u * hp:(u + 1) * hp] = gq[g][:, rows]
                dk[:, held[(g, u2)], u * hkp:(u + 1) * hkp] = gk[g][:, rows]
                dv[:, held[(g, u2)], u * hkp:(u + 1) * hkp] = gv[g][:, rows]
    return dq, dk, dv


def attention_bwd_doc(q, k, v, do, causal, scale, doc_starts, pos_q=None, pos_k=None, nthreads=None):
    """Gradients of attention_doc (the document mask of section All-Gather 式 CP).
    Returns (dq, dk, dv) in float64."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    b, sq, hq, d = q.shape
    _, sk, hkv, _ = k.shape
    if do.shape != q.shape or v.shape != k.shape:
        raise ValueError("shape mismatch")
    pq, pk = _opt_pos(pos_q, sq, "pos_q"), _opt_pos(pos_k, sk, "pos_k")
    docs = _docs(doc_starts)
    dq, dkk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _load().oracle_attention_bwd_doc(_ptr(q, _F64P), _ptr(k, _F64P), _ptr(v, _F64P), _ptr(do, _F64P),
                                          _ptr(pq, _I64P), _ptr(pk, _I64P), b, sq, sk, hq, hkv, d, int(bool(causal)),
                                          _ptr(docs, _I64P), docs.size, float(scale), _ptr(dq, _F64P),
                                          _ptr(dkk, _F64P), _ptr(dv, _F64P), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_attention_bwd_doc rejected its arguments")
    return dq, dkk, dv


def allgather_attention_bwd(q, k, v, do, layout_name, n_ranks, causal, scale, doc_starts, nthreads=None):
    """Reference gradients of All-Gather CP (gathered K/V, document mask; the dK, dV
    reduce-scatter sums every rank's share): the definition over the whole sequence.
    Returns (dq, dk, dv) in ORIGINAL token order."""
    layout.tokens_per_rank(layout_name, n_ranks, q.shape[1])
    return attention_bwd_doc(q, k, v, do, causal, scale, doc_starts, nthreads=nthreads)


def allgather_attention_bwd_steps(q, k, v, do, layout_name, n_ranks, causal, scale, doc_starts, nthreads=None):
    """The All-Gather backward written out: each rank's queries against the gathered
    K/V give its dq and a full-length share of dK, dV; the reduce-scatter sums the
    shares and hands each rank its own block (returned here in original order)."""
    S = q.shape[1]
    layout.tokens_per_rank(layout_name, n_ranks, S)
    q64, do64 = _f64(q), _f64(do)
    o, lse = attention_doc(q, k, v, causal, scale, doc_starts, nthreads=nthreads)
    delta = np.einsum("bshd,bshd->bhs", do64, o)
    dq = np.zeros(q64.shape)
    dk_sum = np.zeros(_f64(k).shape)
    dv_sum = np.zeros(_f64(v).shape)
    docs = _docs(doc_starts)
    for i in range(n_ranks):
        pos = np.asarray(layout.rank_positions(layout_name, n_ranks, S, i), dtype=np.int64)
        # the rank's own share, with the global statistics of its rows: dq rows and a
        # full-length dK, dV contribution (keys of other documents masked)
        q_i, do_i = q64[:, pos], do64[:, pos]
        share = _share_doc(q_i, k, v, do_i, causal, scale, docs, pos, lse[:, :, pos], delta[:, :, pos], nthreads)
        dq[:, pos] = share[0]
        dk_sum += share[1]
        dv_sum += share[2]
    return dq, dk_sum, dv_sum


def _share_doc(q_i, k, v, do_i, causal, scale, docs, pos, lse_i, delta_i, nthreads):
    """One rank's share under the document mask, as a block with global statistics:
    documents cut the keys into independent groups, so the share is summed document
    by document with oracle_attention_bwd's block mode."""
    S = k.shape[1]
    bounds = list(docs) + [S]
    dq = np.zeros(q_i.shape)
    dk = np.zeros(_f64(k).shape)
    dv = np.zeros(_f64(v).shape)
    for a, e in zip(bounds[:-1], bounds[1:]):
        rows = np.nonzero((pos >= a) & (pos < e))[0]
        if rows.size == 0:
            continue
        keys = np.arange(a, e)
        gq, gk, gv, _, _ = attention_bwd(q_i[:, rows], _f64(k)[:, keys], _f64(v)[:, keys], do_i[:, rows], causal,
                                         scale, pos_q=pos[rows], pos_k=keys, lse=lse_i[:, :, rows],
                                         delta=delta_i[:, :, rows], nthreads=nthreads)
        dq[:, rows] = gq
        dk[:, keys] += gk
        dv[:, keys] += gv
    return dq, dk, dv
