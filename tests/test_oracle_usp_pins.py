"""Pins for the oracle's USP form ("DeepSpeed-Ulysses" page, section on USP: Ulysses
inside each group, the ring across groups).  The exchange is a bijection that gives
rank (g, u) exactly the ring block g (the layout's positions, in layout order) for
head group u; with one ring group it is the Ulysses exchange; and the hybrid's
steps (exchange, ring with LSE merges, exchange back) give plain attention and its
gradients."""
import itertools

import numpy as np
import pytest

import oracle
from oracle import layout as L


def _codes(b, S, H, d):
    # every element a distinct integer that names its own (b, s, h, e)
    return np.arange(b * S * H * d, dtype=np.float64).reshape(b, S, H, d)


def _decode(code, S, H, d):
    code = int(code)
    e = code % d
    h = (code // d) % H
    s = (code // (d * H)) % S
    bb = code // (d * H * S)
    return bb, s, h, e


@pytest.mark.parametrize("layout,N,P", [("zigzag", 2, 2), ("striped", 3, 2), ("contiguous", 2, 4), ("zigzag", 1, 4),
                                        ("striped", 4, 1)])
def test_exchange_gives_each_rank_its_ring_block_and_head_group(layout, N, P):
    b, H, d = 2, 8, 2
    S = 2 * N * P * 2
    x = _codes(b, S, H, d)
    out = oracle.usp_exchange(x, layout, N, P)
    hp, c = H // P, S // N
    seen = []
    for (g, u), blk in out.items():
        assert blk.shape == (b, c, hp, d)
        block_pos = L.rank_positions(layout, N, S, g)     # the ring block of group g, layout order
        for bb, t, hh, e in itertools.product(range(b), range(c), range(hp), range(d)):
            got = _decode(blk[bb, t, hh, e], S, H, d)
            assert got == (bb, block_pos[t], u * hp + hh, e), ((g, u), (bb, t, hh, e), got)
        seen.extend(blk.ravel().tolist())
    assert sorted(seen) == x.ravel().tolist()    # a bijection: every element once


def test_one_ring_group_is_the_ulysses_exchange():
    b, S, H, d, P = 2, 16, 8, 3, 4
    x = _codes(b, S, H, d)
    usp = oracle.usp_exchange(x, "contiguous", 1, P)
    uly = oracle.ulysses_all_to_all(x, P)
    for u in range(P):
        assert np.array_equal(usp[(0, u)], uly[u])


CASES = [("zigzag", 2, 2, True), ("striped", 2, 2, True), ("contiguous", 3, 2, True), ("zigzag", 2, 4, False),
         ("striped", 4, 1, True), ("contiguous", 1, 4, True), ("zigzag", 4, 2, True)]


@pytest.mark.parametrize("layout,N,P,causal", CASES)
def test_steps_equal_plain_attention(layout, N, P, causal):
    r = np.random.default_rng(N * 10 + P)
    b, hq, hkv, d = 2, 8, 4, 5
    S = 2 * N * P * 2
    q, k, v = r.standard_normal((b, S, hq, d)), r.standard_normal((b, S, hkv, d)), r.standard_normal((b, S, hkv, d))
    o, lse = oracle.usp_attention_steps(q, k, v, layout, N, P, causal, 0.4)
    ow, lw = oracle.usp_attention(q, k, v, layout, N, P, causal, 0.4)
    assert np.max(np.abs(o - ow)) <= 1e-12
    assert np.max(np.abs(lse - lw)) <= 1e-12


@pytest.mark.parametrize("layout,N,P,causal", CASES[:5])
def test_backward_steps_equal_plain_gradients(layout, N, P, causal):
    r = np.random.default_rng(N * 7 + P)
    b, hq, hkv, d = 1, 8, 4, 3
    S = 2 * N * P * 2
    q, k, v, do = (r.standard_normal(s) for s in ((b, S, hq, d), (b, S, hkv, d), (b, S, hkv, d), (b, S, hq, d)))
    got = oracle.usp_attention_bwd_steps(q, k, v, do, layout, N, P, causal, 0.6)
    want = oracle.usp_attention_bwd(q, k, v, do, layout, N, P, causal, 0.6)
    for g, w in zip(got, want):
        assert np.max(np.abs(g - w)) <= 1e-12


def test_backward_steps_match_finite_differences():
    """An independent pin of the step-by-step gradients: central differences of the
    loss sum(dO . o) through the step-by-step forward."""
    r = np.random.default_rng(5)
    b, S, hq, hkv, d, N, P = 1, 8, 4, 2, 2, 2, 2
    q, k, v, do = (r.standard_normal(s) for s in ((b, S, hq, d), (b, S, hkv, d), (b, S, hkv, d), (b, S, hq, d)))
    dq, dk, dv = oracle.usp_attention_bwd_steps(q, k, v, do, "zigzag", N, P, True, 0.7)

    def loss(qq, kk, vv):
        o, _ = oracle.usp_attention_steps(qq, kk, vv, "zigzag", N, P, True, 0.7, nthreads=1)
        return float(np.sum(o * do))

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 3, 1, 1), (0, 7, x.shape[2] - 1, 0), (0, 5, 0, 1)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-7, (name, idx, fd, g[idx])


def test_shape_conditions():
    x = np.zeros((1, 16, 6, 2))
    with pytest.raises(ValueError):       # 4 does not divide 6 heads
        oracle.usp_attention(x, x[:, :, :2], x[:, :, :2], "zigzag", 2, 4, True, 0.5)
    y = np.zeros((1, 12, 4, 2))
    with pytest.raises(ValueError):       # a ring block of 6 tokens does not split into 4 slices
        oracle.usp_attention_steps(y, y, y, "contiguous", 2, 4, True, 0.5)
