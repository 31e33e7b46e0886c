"""Pins for the oracle's document mask (section All-Gather 式 CP: several documents
packed into one sequence; a key of another document is invisible).

- documents are independent: attention under the mask equals plain attention of
  each document on its own, glued together;
- a pure-Python brute force (math.fsum, no max shift) with the mask on tiny inputs;
- one document is plain attention;
- the All-Gather schedule (each rank's queries against the gathered K/V) equals the
  whole-sequence result for every layout.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import layout as L


def _inputs(seed, b, S, hq, hkv, d):
    r = np.random.default_rng(seed)
    return r.standard_normal((b, S, hq, d)), r.standard_normal((b, S, hkv, d)), r.standard_normal((b, S, hkv, d))


@pytest.mark.parametrize("causal", [True, False])
def test_documents_are_independent(causal):
    b, S, hq, hkv, d = 2, 40, 4, 2, 5
    q, k, v = _inputs(3, b, S, hq, hkv, d)
    starts = [0, 7, 8, 21, 33]
    o, lse = oracle.attention_doc(q, k, v, causal, 0.6, starts)
    bounds = starts + [S]
    for a, e in zip(bounds[:-1], bounds[1:]):
        od, ld = oracle.attention(q[:, a:e], k[:, a:e], v[:, a:e], causal, 0.6)
        assert np.max(np.abs(o[:, a:e] - od)) <= 1e-13
        assert np.max(np.abs(lse[:, :, a:e] - ld)) <= 1e-13


def _brute(q, k, v, causal, scale, starts, pos):
    b, S, hq, d = q.shape
    g = hq // k.shape[2]
    doc = [max(i for i, s0 in enumerate(starts) if s0 <= p) for p in pos]
    o = np.zeros_like(q)
    lse = np.zeros((b, hq, S))
    for bb in range(b):
        for h in range(hq):
            for i in range(S):
                keys = [t for t in range(S) if doc[t] == doc[i] and (not causal or pos[t] <= pos[i])]
                e = {t: math.exp(scale * math.fsum(q[bb, i, h, x] * k[bb, t, h // g, x] for x in range(d)))
                     for t in keys}
                z = math.fsum(e.values())
                for x in range(d):
                    o[bb, i, h, x] = math.fsum(e[t] * v[bb, t, h // g, x] for t in keys) / z
                lse[bb, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("causal", [True, False])
def test_doc_mask_brute_force_with_permuted_positions(causal):
    b, S, hq, hkv, d = 1, 12, 2, 1, 3
    q, k, v = _inputs(9, b, S, hq, hkv, d)
    pos = np.array(L.rank_positions("zigzag", 2, S, 1) + L.rank_positions("zigzag", 2, S, 0))
    starts = [0, 4, 5, 9]
    o, lse = oracle.attention_doc(q, k, v, causal, 0.7, starts, pos_q=pos, pos_k=pos)
    ob, lb = _brute(q, k, v, causal, 0.7, starts, pos)
    assert np.max(np.abs(o - ob)) <= 1e-13
    assert np.max(np.abs(lse - lb)) <= 1e-13


def test_one_document_is_plain_attention():
    q, k, v = _inputs(4, 1, 24, 4, 2, 6)
    o, lse = oracle.attention_doc(q, k, v, True, 0.5, [0])
    o2, l2 = oracle.attention(q, k, v, True, 0.5)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N", [2, 4])
def test_allgather_schedule_equals_whole(layout, N):
    S = 32
    q, k, v = _inputs(N + len(layout), 2, S, 4, 2, 4)
    starts = [0, 3, 16, 17, 30]
    want = oracle.allgather_attention(q, k, v, layout, N, True, 0.4, starts)
    got = oracle.allgather_attention_steps(q, k, v, layout, N, True, 0.4, starts)
    assert np.max(np.abs(got[0] - want[0])) <= 1e-13
    assert np.max(np.abs(got[1] - want[1])) <= 1e-13


def test_rows_doc_matches_full():
    q, k, v = _inputs(6, 2, 30, 4, 2, 5)
    starts = [0, 11, 12, 25]
    o, lse = oracle.attention_doc(q, k, v, True, 0.3, starts)
    sel = np.array([[0, 0, 0], [1, 3, 11], [0, 2, 29], [1, 1, 12], [0, 1, 24]])
    os_, ls = oracle.attention_rows_doc(np.stack([q[b, p, h] for b, h, p in sel]), sel, k, v, True, 0.3, 4, starts)
    for r, (b, h, p) in enumerate(sel):
        assert np.max(np.abs(os_[r] - o[b, p, h])) <= 1e-14
        assert abs(ls[r] - lse[b, h, p]) <= 1e-14


def test_doc_starts_are_checked():
    q, k, v = _inputs(1, 1, 8, 2, 1, 2)
    for bad in ([1, 4], [0, 4, 4], [0, 5, 3]):
        with pytest.raises(ValueError):
            oracle.attention_doc(q, k, v, True, 0.5, bad)


# ------------------------------------------------------------------ backward

def _loss_doc(q, k, v, do, causal, scale, starts, pos):
    o, _ = oracle.attention_doc(q, k, v, causal, scale, starts, pos_q=pos, pos_k=pos, nthreads=1)
    return float(np.sum(o * do))


def test_doc_gradients_match_finite_differences():
    b, S, hq, hkv, d = 1, 9, 2, 1, 3
    q, k, v = _inputs(12, b, S, hq, hkv, d)
    do = np.random.default_rng(13).standard_normal(q.shape)
    pos = np.array(L.rank_positions("zigzag", 3, 18, 1) + L.rank_positions("zigzag", 3, 18, 2)[:3])
    starts = [0, 4, 11, 15]
    dq, dk, dv = oracle.attention_bwd_doc(q, k, v, do, True, 0.9, starts, pos_q=pos, pos_k=pos)
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + 1e-5
            fp = _loss_doc(q, k, v, do, True, 0.9, starts, pos)
            x[idx] = old - 1e-5
            fm = _loss_doc(q, k, v, do, True, 0.9, starts, pos)
            x[idx] = old
            num[idx] = (fp - fm) / 2e-5
        assert np.max(np.abs(num - g)) <= 1e-7


def test_doc_gradients_are_per_document():
    b, S, hq, hkv, d = 2, 30, 4, 2, 4
    q, k, v = _inputs(14, b, S, hq, hkv, d)
    do = np.random.default_rng(15).standard_normal(q.shape)
    starts = [0, 9, 10, 22]
    dq, dk, dv = oracle.attention_bwd_doc(q, k, v, do, True, 0.5, starts)
    bounds = starts + [S]
    for a, e in zip(bounds[:-1], bounds[1:]):
        gq, gk, gv, _, _ = oracle.attention_bwd(q[:, a:e], k[:, a:e], v[:, a:e], do[:, a:e], True, 0.5)
        assert np.max(np.abs(dq[:, a:e] - gq)) <= 1e-13
        assert np.max(np.abs(dk[:, a:e] - gk)) <= 1e-13
        assert np.max(np.abs(dv[:, a:e] - gv)) <= 1e-13


@pytest.mark.parametrize("layout", L.LAYOUTS)
def test_allgather_backward_steps_equal_whole(layout):
    S, N = 32, 4
    q, k, v = _inputs(16 + len(layout), 1, S, 4, 2, 3)
    do = np.random.default_rng(17).standard_normal(q.shape)
    starts = [0, 5, 6, 19, 31]
    got = oracle.allgather_attention_bwd_steps(q, k, v, do, layout, N, True, 0.4, starts)
    want = oracle.allgather_attention_bwd(q, k, v, do, layout, N, True, 0.4, starts)
    for g, w in zip(got, want):
        assert np.max(np.abs(g - w)) <= 1e-12
