"""Pins for the oracle's gradients: each test checks them against something other
than the gradient code itself.

Source: "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力, the
paragraph on the backward pass (p_j = e^{x_j - lse} with the global lse,
dv_j = sum p_j do, dx_j = p_j (do . v_j - D), D = do . o), and section Ring
Attention (at step r rank i holds the K/V of rank (i - r) mod N).

- central finite differences of the oracle's FORWARD (loss sum(do * o)) fix every
  term, sign, index and the GQA head sum of dq, dk, dv;
- the step-by-step ring (block shares with the global statistics, dK/dV carried
  with their block) must reproduce the whole-sequence gradients;
- closed forms: uniform attention (q = 0) turns dq into a covariance and dk into
  zero; a row that sees one key has dq = 0;
- invariants: sum_j dk_j = 0 and sum_j dv_j = sum of do over rows that see a key.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import layout as L


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, b, sq, sk, hq, hkv, d):
    r = _rng(seed)
    return (r.standard_normal((b, sq, hq, d)), r.standard_normal((b, sk, hkv, d)),
            r.standard_normal((b, sk, hkv, d)), r.standard_normal((b, sq, hq, d)))


def _loss(q, k, v, do, causal, scale, pos_q, pos_k):
    o, _ = oracle.attention(q, k, v, causal, scale, pos_q=pos_q, pos_k=pos_k, nthreads=1)
    return float(np.sum(o * do))


def _numeric_grad(x, f, h=1e-5):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + h
        fp = f()
        x[idx] = old - h
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("causal", [True, False])
def test_gradients_match_finite_differences(causal):
    b, sq, sk, hq, hkv, d = 2, 5, 6, 4, 2, 3
    q, k, v, do = _inputs(17 + causal, b, sq, sk, hq, hkv, d)
    r = _rng(3)
    pos_q = r.permutation(9)[:sq]
    pos_k = r.permutation(9)[:sk]
    pos_q[0] = -1  # sees no key under the causal mask
    scale = 0.8
    dq, dk, dv, lse, _ = oracle.attention_bwd(q, k, v, do, causal, scale, pos_q=pos_q, pos_k=pos_k, nthreads=2)
    f = lambda: _loss(q, k, v, do, causal, scale, pos_q, pos_k)  # noqa: E731
    for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv)):
        num = _numeric_grad(x, f)
        err = np.max(np.abs(num - g))
        assert err <= 1e-7 * max(1.0, np.max(np.abs(num))), (name, err)
    if causal:
        assert np.all(lse[:, :, 0] == -np.inf) and np.all(dq[:, 0] == 0.0)


def test_finite_differences_with_identity_positions_and_mha():
    q, k, v, do = _inputs(5, 1, 7, 7, 2, 2, 4)
    dq, dk, dv, _, _ = oracle.attention_bwd(q, k, v, do, True, 0.5)
    f = lambda: _loss(q, k, v, do, True, 0.5, None, None)  # noqa: E731
    for x, g in ((q, dq), (k, dk), (v, dv)):
        assert np.max(np.abs(_numeric_grad(x, f) - g)) <= 1e-7


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,causal", [(2, True), (4, True), (4, False), (1, True)])
def test_ring_steps_reproduce_whole_gradients(layout, N, causal):
    S = 16
    q, k, v, do = _inputs(N * 7 + len(layout), 2, S, S, 4, 2, 5)
    want = oracle.ring_attention_bwd(q, k, v, do, layout, N, causal, 0.45)
    got = oracle.ring_attention_bwd_steps(q, k, v, do, layout, N, causal, 0.45)
    for g, w in zip(got, want):
        assert np.max(np.abs(g - w)) <= 1e-12 * max(1.0, np.max(np.abs(w)))


def test_block_share_with_global_statistics_sums_to_whole():
    """Two arbitrary key blocks (positions interleaved) with the global (lse, D):
    their dq shares add up to the whole dq; dk, dv are the blocks' rows."""
    q, k, v, do = _inputs(21, 1, 10, 12, 2, 1, 4)
    pos_q = np.arange(2, 12)
    pos_k = np.arange(12)
    dq, dk, dv, lse, delta = oracle.attention_bwd(q, k, v, do, True, 0.6, pos_q=pos_q, pos_k=pos_k)
    blk = [np.array([0, 3, 4, 9, 10]), np.array([1, 2, 5, 6, 7, 8, 11])]
    acc = np.zeros_like(dq)
    for ids in blk:
        gq, gk, gv, _, _ = oracle.attention_bwd(q, k[:, ids], v[:, ids], do, True, 0.6, pos_q=pos_q,
                                                pos_k=pos_k[ids], lse=lse, delta=delta)
        acc += gq
        assert np.max(np.abs(gk - dk[:, ids])) <= 1e-13
        assert np.max(np.abs(gv - dv[:, ids])) <= 1e-13
    assert np.max(np.abs(acc - dq)) <= 1e-13


@pytest.mark.parametrize("causal", [True, False])
def test_uniform_attention_closed_form(causal):
    """q = 0: every visible key has p = 1/n, so dk = 0, dv_j = sum_i do_i / n_i and
    dq_i = scale * Cov_i(k, v) do_i, the covariance over the keys row i sees."""
    b, S, hq, hkv, d = 1, 9, 2, 1, 3
    _, k, v, do = _inputs(8, b, S, S, hq, hkv, d)
    q = np.zeros((b, S, hq, d))
    scale = 0.7
    dq, dk, dv, _, _ = oracle.attention_bwd(q, k, v, do, causal, scale)
    assert np.max(np.abs(dk)) <= 1e-14
    want_dv = np.zeros_like(dv)
    want_dq = np.zeros_like(dq)
    for h in range(hq):
        for i in range(S):
            keys = list(range(i + 1)) if causal else list(range(S))
            n = len(keys)
            kk, vv = k[0, keys, 0], v[0, keys, 0]
            for t in keys:
                want_dv[0, t, 0] += do[0, i, h] / n
            cov = (kk - kk.mean(0)).T @ (vv - vv.mean(0)) / n  # [d_k, d_v]
            want_dq[0, i, h] = scale * cov @ do[0, i, h]
    assert np.max(np.abs(dv - want_dv)) <= 1e-13
    assert np.max(np.abs(dq - want_dq)) <= 1e-13


def test_row_with_one_visible_key_has_zero_dq():
    q, k, v, do = _inputs(9, 1, 6, 6, 2, 2, 4)
    dq, _, _, _, _ = oracle.attention_bwd(q, k, v, do, True, 0.5)
    assert np.max(np.abs(dq[:, 0])) <= 1e-15
    assert np.max(np.abs(dq[:, 1:])) > 1e-3


@pytest.mark.parametrize("causal", [True, False])
def test_gradient_sums(causal):
    """sum_j dx_j = 0 per row (the probabilities sum to 1), hence sum_j dk_j = 0;
    sum_j dv_j = sum over the group's rows that see a key of do."""
    b, S, hq, hkv, d = 2, 24, 6, 2, 5
    q, k, v, do = _inputs(33, b, S, S, hq, hkv, d)
    pos = np.asarray(L.rank_positions("zigzag", 3, S, 1) + L.rank_positions("zigzag", 3, S, 0)
                     + L.rank_positions("zigzag", 3, S, 2))
    _, dk, dv, lse, _ = oracle.attention_bwd(q, k, v, do, causal, 0.4, pos_q=pos, pos_k=pos)
    g = hq // hkv
    for bb in range(b):
        for hk in range(hkv):
            assert np.max(np.abs(dk[bb, :, hk].sum(0))) <= 1e-12
            heads = range(hk * g, (hk + 1) * g)
            want = sum(do[bb, i, h] for h in heads for i in range(S) if np.isfinite(lse[bb, h, i]))
            assert np.max(np.abs(dv[bb, :, hk].sum(0) - want)) <= 1e-12


def test_key_shift_leaves_gradients_unchanged():
    """Adding one vector to every key shifts a row's scores by a constant: the
    softmax, hence o and every gradient, is unchanged."""
    q, k, v, do = _inputs(44, 1, 8, 8, 2, 1, 4)
    c = np.array([0.3, -1.2, 0.5, 2.0])
    a = oracle.attention_bwd(q, k, v, do, True, 0.5)
    b_ = oracle.attention_bwd(q, k + c, v, do, True, 0.5)
    for x, y in zip(a[:3], b_[:3]):
        assert np.max(np.abs(x - y)) <= 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_selected_rows_match_full(causal):
    b, S, hq, hkv, d = 2, 20, 4, 2, 6
    q, k, v, do = _inputs(55, b, S, S, hq, hkv, d)
    pos = np.asarray(L.rank_positions("striped", 4, S, 2) + L.rank_positions("striped", 4, S, 0)
                     + L.rank_positions("striped", 4, S, 3) + L.rank_positions("striped", 4, S, 1))
    dq, dk, dv, _, _ = oracle.attention_bwd(q, k, v, do, causal, 0.3, pos_q=pos, pos_k=pos)
    sel_q = np.array([[0, 0, 0], [1, 3, 19], [0, 2, 7], [1, 1, 11]])
    sel_k = np.array([[0, 0, 0], [1, 1, 19], [0, 1, 5], [1, 0, 12]])
    gq, gk, gv = oracle.attention_bwd_sel(q, k, v, do, causal, 0.3, sel_q, sel_k, pos_q=pos, pos_k=pos)
    for r, (bb, h, i) in enumerate(sel_q):
        assert np.max(np.abs(gq[r] - dq[bb, i, h])) <= 1e-14
    for r, (bb, hk, t) in enumerate(sel_k):
        assert np.max(np.abs(gk[r] - dk[bb, t, hk])) <= 1e-14
        assert np.max(np.abs(gv[r] - dv[bb, t, hk])) <= 1e-14


def test_bwd_rejects_bad_arguments():
    q, k, v, do = _inputs(1, 1, 4, 4, 3, 2, 2)
    with pytest.raises(ValueError):
        oracle.attention_bwd(q, k, v, do, True, 0.5)  # hq % hkv
    q, k, v, do = _inputs(1, 1, 4, 4, 2, 1, 2)
    with pytest.raises(ValueError):
        oracle.attention_bwd(q, k, v, do[:, :3], True, 0.5)
    with pytest.raises(ValueError):
        oracle.attention_bwd_sel(q, k, v, do, True, 0.5, [[0, 2, 0]], [])
    with pytest.raises(ValueError):
        oracle.attention_bwd_sel(q, k, v, do, True, 0.5, [], [[0, 0, 4]])
    assert math.isfinite(oracle.attention_bwd(q, k, v, do, True, 0.5)[0].sum())
