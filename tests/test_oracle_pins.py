"""Pins for the fp64 oracle: each test checks it against something other than itself.

Sources: "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力
(softmax definition, per-block statistics, boxed merge identity, stable form,
weights summing to 1, the 8-key two-block example), section 因果掩码带来的负载不均
(causal mask on positions) and the Llama-3 GQA head table on the tensor-parallel
page (several query heads share one KV head).
"""
import itertools
import math

import numpy as np
import pytest

import oracle


def _bruteforce(q, k, v, causal, scale, pos_q=None, pos_k=None):
    """Independent pure-Python softmax without any max shift, summed with math.fsum."""
    b, sq, hq, d = q.shape
    _, sk, hkv, _ = k.shape
    group = hq // hkv
    pos_q = list(range(sq)) if pos_q is None else list(pos_q)
    pos_k = list(range(sk)) if pos_k is None else list(pos_k)
    o = np.zeros((b, sq, hq, d))
    lse = np.zeros((b, hq, sq))
    for bb in range(b):
        for h in range(hq):
            kh = h // group
            for s in range(sq):
                keys = [t for t in range(sk) if (not causal) or pos_k[t] <= pos_q[s]]
                if not keys:
                    lse[bb, h, s] = -math.inf
                    continue
                e = {t: math.exp(scale * math.fsum(float(q[bb, s, h, i]) * float(k[bb, t, kh, i])
                                                   for i in range(d))) for t in keys}
                z = math.fsum(e.values())
                for i in range(d):
                    o[bb, s, h, i] = math.fsum(e[t] * float(v[bb, t, kh, i]) for t in keys) / z
                lse[bb, h, s] = math.log(z)
    return o, lse


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", [(1, 7, 2, 2, 5), (2, 16, 4, 2, 3), (1, 9, 3, 1, 4)])
def test_bruteforce_direct_softmax(causal, shape):
    b, S, hq, hkv, d = shape
    r = _rng(S * 31 + hq)
    q = r.standard_normal((b, S, hq, d))
    k = r.standard_normal((b, S, hkv, d))
    v = r.standard_normal((b, S, hkv, d))
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention(q, k, v, causal, scale)
    ob, lb = _bruteforce(q, k, v, causal, scale)
    assert np.max(np.abs(o - ob)) <= 1e-13
    assert np.max(np.abs(lse - lb)) <= 1e-13


def test_bruteforce_with_permuted_positions():
    """Masking on original positions, not on storage order (section 重排 token 的代价)."""
    r = _rng(5)
    b, sq, sk, hq, hkv, d = 1, 6, 8, 2, 1, 4
    q = r.standard_normal((b, sq, hq, d))
    k = r.standard_normal((b, sk, hkv, d))
    v = r.standard_normal((b, sk, hkv, d))
    pos_q = r.permutation(12)[:sq]
    pos_k = r.permutation(12)[:sk]
    o, lse = oracle.attention(q, k, v, True, 0.37, pos_q=pos_q, pos_k=pos_k)
    ob, lb = _bruteforce(q, k, v, True, 0.37, pos_q, pos_k)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - lb[fin])) <= 1e-13
    assert np.max(np.abs(o - ob)) <= 1e-13


def test_large_scores_need_the_max_shift():
    """Scores near 800 overflow exp() unless the max is subtracted (m_b in the page)."""
    q = np.full((1, 3, 1, 2), 20.0)
    k = np.array([[[[20.0, 20.0]], [[19.5, 20.0]], [[20.0, 19.0]]]])
    v = np.arange(6, dtype=np.float64).reshape(1, 3, 1, 2)
    o, lse = oracle.attention(q, k, v, False, 1.0)
    x = [800.0, 790.0, 780.0]
    m = max(x)
    w = [math.exp(t - m) for t in x]
    z = math.fsum(w)
    for s in range(3):
        assert abs(lse[0, 0, s] - (m + math.log(z))) <= 1e-12
        for i in range(2):
            ref = math.fsum(w[t] * v[0, t, 0, i] for t in range(3)) / z
            assert abs(o[0, s, 0, i] - ref) <= 1e-13


def test_q_zero_gives_log_count_and_mean():
    """Q = 0: every score is 0, so lse = log |K(p)| and o is the mean of visible values."""
    r = _rng(11)
    b, S, hq, hkv, d = 2, 13, 4, 2, 6
    q = np.zeros((b, S, hq, d))
    k = r.standard_normal((b, S, hkv, d))
    v = r.standard_normal((b, S, hkv, d))
    o, lse = oracle.attention(q, k, v, True, 0.125)
    for p in range(S):
        assert np.allclose(lse[:, :, p], math.log(p + 1), atol=1e-14, rtol=0)
        for h in range(hq):
            mean = v[:, : p + 1, h // 2, :].mean(axis=1)
            assert np.max(np.abs(o[:, p, h, :] - mean)) <= 1e-14
    o2, lse2 = oracle.attention(q, k, v, False, 0.125)
    assert np.allclose(lse2, math.log(S), atol=1e-14, rtol=0)


def test_first_position_sees_only_itself():
    """Causal position 0: o = v_0 and lse = x_0 = scale * q_0 . k_0."""
    r = _rng(3)
    q = r.standard_normal((1, 5, 2, 8))
    k = r.standard_normal((1, 5, 2, 8))
    v = r.standard_normal((1, 5, 2, 8))
    scale = 1.0 / math.sqrt(8)
    o, lse = oracle.attention(q, k, v, True, scale)
    for h in range(2):
        assert np.max(np.abs(o[0, 0, h] - v[0, 0, h])) == 0.0
        x0 = scale * math.fsum(q[0, 0, h, i] * k[0, 0, h, i] for i in range(8))
        assert abs(lse[0, h, 0] - x0) <= 1e-14


def test_identical_keys_average_values():
    r = _rng(4)
    S, d = 10, 3
    q = r.standard_normal((1, S, 1, d))
    krow = r.standard_normal(d)
    k = np.broadcast_to(krow, (1, S, 1, d)).copy()
    v = r.standard_normal((1, S, 1, d))
    o, lse = oracle.attention(q, k, v, True, 0.5)
    for p in range(S):
        assert np.max(np.abs(o[0, p, 0] - v[0, : p + 1, 0].mean(axis=0))) <= 1e-14
        x = 0.5 * float(q[0, p, 0] @ krow)
        assert abs(lse[0, 0, p] - (x + math.log(p + 1))) <= 1e-13


def test_gqa_head_grouping():
    """Query head h reads KV head h // (Hq/Hkv): with V constant per KV head the
    output names the KV head it came from."""
    r = _rng(8)
    b, S, hq, hkv, d = 1, 6, 8, 2, 4
    q = r.standard_normal((b, S, hq, d))
    k = r.standard_normal((b, S, hkv, d))
    v = np.zeros((b, S, hkv, d))
    for j in range(hkv):
        v[:, :, j, :] = j + 1.0
    o, _ = oracle.attention(q, k, v, True, 0.5)
    for h in range(hq):
        assert np.allclose(o[:, :, h, :], h // (hq // hkv) + 1.0, atol=1e-14, rtol=0)


def test_rows_mode_matches_full():
    r = _rng(9)
    b, S, hq, hkv, d = 2, 12, 4, 2, 8
    q = r.standard_normal((b, S, hq, d))
    k = r.standard_normal((b, S, hkv, d))
    v = r.standard_normal((b, S, hkv, d))
    o, lse = oracle.attention(q, k, v, True, 0.3)
    sel = np.array([[0, 0, 0], [1, 3, 11], [0, 2, 5], [1, 1, 7]])
    q_sel = np.stack([q[bb, s, h] for bb, h, s in sel])
    os_, ls_ = oracle.attention_rows(q_sel, sel, k, v, True, 0.3, hq)
    for n, (bb, h, s) in enumerate(sel):
        assert np.array_equal(os_[n], o[bb, s, h])
        assert ls_[n] == lse[bb, h, s]


# ------------------------------------------------------------------------- merge


def _partial(qv, keys, vals, idx, scale):
    """Oracle partial (o_b, lse_b) of one query over the key subset idx."""
    k = keys[idx][None, :, None, :]
    v = vals[idx][None, :, None, :]
    o, lse = oracle.attention(qv[None, None, None, :], k, v, False, scale)
    return o[0, 0, 0], lse[0, 0, 0]


def test_eight_keys_every_two_block_split():
    """One query, 8 keys with 2-D values split into two blocks (the page's figure):
    merging the two partials with the boxed formula gives one-shot softmax, for
    every unordered split into two nonempty sets and every contiguous split."""
    r = _rng(21)
    d = 2
    qv = r.standard_normal(d) * 2.0
    keys = r.standard_normal((8, d)) * 2.0
    vals = r.standard_normal((8, d))
    full_o, full_lse = _partial(qv, keys, vals, list(range(8)), 1 / math.sqrt(d))
    splits = []
    for mask in range(1, 255):
        if mask & 1:  # one representative of each unordered pair
            splits.append([t for t in range(8) if mask >> t & 1])
    assert len(splits) == 127
    splits += [list(range(c)) for c in range(1, 8)]
    for b1 in splits:
        b2 = [t for t in range(8) if t not in b1]
        o1, l1 = _partial(qv, keys, vals, b1, 1 / math.sqrt(d))
        o2, l2 = _partial(qv, keys, vals, b2, 1 / math.sqrt(d))
        for (oa, la, ob, lb) in ((o1, l1, o2, l2), (o2, l2, o1, l1)):
            o, lse = oracle.lse_merge(oa[None], np.array([la]), ob[None], np.array([lb]))
            assert np.max(np.abs(o[0] - full_o)) <= 1e-12
            assert abs(lse[0] - full_lse) <= 1e-12
            # the boxed identity written directly: lse = log(e^lse1 + e^lse2)
            assert abs(lse[0] - math.log(math.exp(la) + math.exp(lb))) <= 1e-12


def test_many_block_splits_merged_in_any_order():
    """The ring folds N partials one after the other, in its own step order.  For
    random partitions of up to 64 keys into up to 8 nonempty blocks (some empty
    blocks too, lse = -inf), merging the blocks' partials one by one in a random
    order, starting from the empty accumulator (0, -inf), gives one-shot softmax
    (section 分块注意力: the split result equals the unsplit one, for any split)."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=150, deadline=None)
    @given(n=st.integers(1, 64), nb=st.integers(1, 8), seed=st.integers(0, 2 ** 31 - 1))
    def check(n, nb, seed):
        r = np.random.default_rng(seed)
        d = 3
        qv = r.standard_normal(d) * 2.0
        keys = r.standard_normal((n, d)) * 2.0
        vals = r.standard_normal((n, d))
        scale = 1 / math.sqrt(d)
        full_o, full_lse = _partial(qv, keys, vals, list(range(n)), scale)
        owner = r.integers(0, nb, n)           # block of each key; a block may stay empty
        order = r.permutation(nb)
        acc_o, acc_l = np.zeros((1, d)), np.array([-np.inf])
        for blk in order:
            idx = [t for t in range(n) if owner[t] == blk]
            if idx:
                ob, lb = _partial(qv, keys, vals, idx, scale)
            else:
                ob, lb = np.zeros(d), -np.inf
            acc_o, acc_l = oracle.lse_merge(acc_o, acc_l, ob[None], np.array([lb]))
        assert np.max(np.abs(acc_o[0] - full_o)) <= 1e-12
        assert abs(acc_l[0] - full_lse) <= 1e-12

    check()


def test_merge_weights_sum_to_one():
    """o_1 = o_2 = 1 returns e^{lse_1-lse} + e^{lse_2-lse}, which must be 1; o_1 = 1,
    o_2 = 0 returns the first weight, e^{lse_1} / (e^{lse_1} + e^{lse_2})."""
    r = _rng(1)
    n = 1000
    l1 = r.uniform(-50, 50, n)
    l2 = l1 + r.uniform(-30, 30, n)
    ones = np.ones((n, 1))
    o, lse = oracle.lse_merge(ones, l1, ones, l2)
    assert np.max(np.abs(o - 1.0)) <= 1e-14
    o, _ = oracle.lse_merge(ones, l1, np.zeros((n, 1)), l2)
    w1 = 1.0 / (1.0 + np.exp(l2 - l1))
    assert np.max(np.abs(o[:, 0] - w1)) <= 1e-14
    assert np.all(lse >= np.maximum(l1, l2))
    assert np.all(lse <= np.maximum(l1, l2) + math.log(2) + 1e-14)


def test_merge_with_empty_partials():
    """An empty partial (lse = -inf) leaves the other unchanged; two empties stay empty."""
    r = _rng(2)
    o2 = r.standard_normal((4, 3))
    l2 = r.standard_normal(4)
    ninf = np.full(4, -np.inf)
    o, lse = oracle.lse_merge(np.zeros((4, 3)), ninf, o2, l2)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)
    o, lse = oracle.lse_merge(o2, l2, np.zeros((4, 3)), ninf)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)
    o, lse = oracle.lse_merge(np.zeros((4, 3)), ninf, np.zeros((4, 3)), ninf)
    assert np.all(o == 0) and np.all(lse == -np.inf)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
def test_ring_of_block_partials_equals_full_attention(layout):
    """Running the ring on the oracle's own block partials (rank i merges the partial
    against rank (i - r) mod N at step r) reproduces full attention in original order."""
    from oracle import layout as L
    r = _rng(17)
    b, S, hq, hkv, d, N = 1, 24, 4, 2, 4, 3
    q = r.standard_normal((b, S, hq, d))
    k = r.standard_normal((b, S, hkv, d))
    v = r.standard_normal((b, S, hkv, d))
    full_o, full_lse = oracle.attention(q, k, v, True, 0.4)
    for i in range(N):
        pq = np.array(L.rank_positions(layout, N, S, i))
        acc_o = np.zeros((b, len(pq), hq, d))
        acc_l = np.full((b, hq, len(pq)), -np.inf)
        for step in range(N):
            j = L.ring_source(i, step, N)
            pk = np.array(L.rank_positions(layout, N, S, j))
            ob, lb = oracle.attention(q[:, pq], k[:, pk], v[:, pk], True, 0.4, pos_q=pq, pos_k=pk)
            mo, ml = oracle.lse_merge(acc_o.transpose(0, 2, 1, 3), acc_l,
                                      ob.transpose(0, 2, 1, 3), lb)
            acc_o, acc_l = mo.transpose(0, 2, 1, 3), ml
        assert np.max(np.abs(acc_o - full_o[:, pq])) <= 1e-12
        assert np.max(np.abs(acc_l - full_lse[:, :, pq])) <= 1e-12
