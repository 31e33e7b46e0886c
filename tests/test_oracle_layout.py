"""Pins for the oracle's integer layout maps and mask enumeration.

Source: "上下文并行与 Ring Attention" (hs-black.github.io): section Ring Attention
(rank i holds rank (i - r) mod N's K/V at step r), section 因果掩码带来的负载不均
(contiguous split, eta_naive), section Zig-zag (2N chunks, the case table, the
per-card work figure, the unmasked-rectangle remark), section Striped (token p on
rank p mod N, causal mask with an offset) and section 重排 token 的代价 (the mask
uses original positions; the layouts are permutations).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import layout as L

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S", [(1, 8), (2, 8), (3, 12), (4, 64), (8, 64)])
def test_layouts_are_permutations(layout, N, S):
    order = L.rank_order(layout, N, S)
    assert sorted(order) == list(range(S))
    if N == 1:
        assert order == list(range(S))
    x = np.arange(2 * S * 3).reshape(2, S, 3)
    xr = L.permute(x, layout, N, axis=1)
    assert np.array_equal(L.unpermute(xr, layout, N, axis=1), x)


def test_layout_maps_by_hand():
    # contiguous: rank i holds i*c .. i*c+c-1
    assert L.rank_positions("contiguous", 4, 16, 2) == [8, 9, 10, 11]
    # zig-zag N=4: chunks of 2; rank 0 holds C_0 and C_7, rank 3 the two middle chunks
    assert L.rank_positions("zigzag", 4, 16, 0) == [0, 1, 14, 15]
    assert L.rank_positions("zigzag", 4, 16, 3) == [6, 7, 8, 9]
    # striped: token p on rank p mod N
    assert L.rank_positions("striped", 4, 16, 1) == [1, 5, 9, 13]


def test_shape_rules():
    with pytest.raises(ValueError):
        L.tokens_per_rank("contiguous", 3, 10)
    with pytest.raises(ValueError):
        L.tokens_per_rank("zigzag", 4, 12)  # 12 % 8 != 0
    assert L.tokens_per_rank("striped", 4, 12) == 3


@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
def test_ring_visits_every_source_once(N):
    for i in range(N):
        srcs = [L.ring_source(i, r, N) for r in range(N)]
        assert sorted(srcs) == list(range(N))
        assert srcs[0] == i
        # at each step every rank holds a different block (a permutation of ranks)
    for r in range(N):
        assert sorted(L.ring_source(i, r, N) for i in range(N)) == list(range(N))


def _closed_form(layout, c, i, j):
    if layout == "contiguous":
        return c * (c + 1) // 2 if j == i else (c * c if j < i else 0)
    if layout == "zigzag":
        return c * c // 2 + c // 2 if j == i else c * c // 2
    return c * (c + 1) // 2 if j <= i else c * (c - 1) // 2  # striped


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S", [(2, 16), (3, 24), (4, 64), (8, 64)])
def test_visible_pairs_per_step_closed_forms(layout, N, S):
    c = S // N
    for i in range(N):
        for r in range(N):
            j = L.ring_source(i, r, N)
            assert L.visible_pairs(layout, N, S, i, j) == _closed_form(layout, c, i, j)
    total = sum(L.visible_pairs(layout, N, S, i, j) for i in range(N) for j in range(N))
    assert total == S * (S + 1) // 2


@pytest.mark.parametrize("N,S", [(2, 8), (4, 32), (5, 20)])
def test_striped_offset_mask(N, S):
    """Striped: local query a on rank i sees local key b on rank j iff b < a, or
    b == a and j <= i (a causal mask whose diagonal depends on the rank pair)."""
    c = S // N
    for i in range(N):
        for j in range(N):
            pq = L.rank_positions("striped", N, S, i)
            pk = L.rank_positions("striped", N, S, j)
            for a in range(c):
                for b in range(c):
                    assert (pk[b] <= pq[a]) == (b < a or (b == a and j <= i))


def test_zigzag_case_table_golden():
    rows = _golden_lines("zigzag_case_table.txt")
    table = {(r[0], r[1]): r[3:6] for r in rows}
    for N in (2, 3, 4, 6):
        for i in range(N):
            for j in range(N):
                q_chunks = {"early": i, "late": 2 * N - 1 - i}
                k_chunks = {"early": j, "late": 2 * N - 1 - j}
                col = 0 if j < i else (1 if j == i else 2)
                for (qn, kn), rule in table.items():
                    got = L.chunk_pair_kind(N, q_chunks[qn], k_chunks[kn])
                    assert got == rule[col], (N, i, j, qn, kn)


@pytest.mark.parametrize("N", [2, 4, 8])
def test_zigzag_two_full_two_skipped_off_diagonal(N):
    for i in range(N):
        for j in range(N):
            kinds = [L.chunk_pair_kind(N, qc, kc) for qc in (i, 2 * N - 1 - i)
                     for kc in (j, 2 * N - 1 - j)]
            if j != i:
                assert sorted(kinds) == ["full", "full", "skip", "skip"]
            else:
                assert sorted(kinds) == ["diag", "diag", "full", "skip"]


@pytest.mark.parametrize("N,S", [(4, 32), (3, 36)])
def test_zigzag_off_diagonal_steps_are_unmasked_rectangles(N, S):
    """j < i: all of Q against the first half of rank j's K/V; j > i: the second
    half of Q against all of rank j's K/V; both dense."""
    c = S // N
    h = c // 2
    for i in range(N):
        for j in range(N):
            if i == j:
                continue
            pq = L.rank_positions("zigzag", N, S, i)
            pk = L.rank_positions("zigzag", N, S, j)
            vis = {(a, b) for a in range(c) for b in range(c) if pk[b] <= pq[a]}
            if j < i:
                assert vis == {(a, b) for a in range(c) for b in range(h)}
            else:
                assert vis == {(a, b) for a in range(h, c) for b in range(c)}


def test_zigzag_work_figure_golden():
    gold = {r[0]: [int(x) for x in r[1:]] for r in _golden_lines("zigzag_work_n4.txt")}
    N = 4
    weight = {"full": Fraction(1), "diag": Fraction(1, 2), "skip": Fraction(0)}
    # contiguous: rank i holds chunks 2i, 2i+1; zig-zag: chunks i, 2N-1-i
    holdings = {"contiguous": [(2 * i, 2 * i + 1) for i in range(N)],
                "zigzag": [(i, 2 * N - 1 - i) for i in range(N)]}
    for name, hold in holdings.items():
        work = [sum(weight[L.chunk_pair_kind(N, qc, kc)] for qc in chunks
                    for kc in range(2 * N)) for chunks in hold]
        assert work == gold[name], name


def test_naive_efficiency_golden():
    gold = {int(r[0]): int(r[1]) for r in _golden_lines("naive_efficiency.txt")}
    for N, pct in gold.items():
        assert round(100 * N / (2 * N - 1)) == pct
        # the element-exact efficiency from brute-force per-step counts: the slowest
        # rank sets each step's time
        c = 16
        S = N * c
        useful = sum(L.visible_pairs("contiguous", N, S, i, j) for i in range(N) for j in range(N))
        busiest = sum(max(L.visible_pairs("contiguous", N, S, i, L.ring_source(i, r, N))
                          for i in range(N)) for r in range(N))
        eta = Fraction(useful, N * busiest)
        exact = Fraction(N * c * (c + 1) // 2 + N * (N - 1) * c * c // 2,
                         N * (c * (c + 1) // 2 + (N - 1) * c * c))
        assert eta == exact
        assert abs(float(eta) - N / (2 * N - 1)) < 1.0 / c
    # zig-zag and striped balance: every step costs the same on every rank but step 0
    for layout in ("zigzag", "striped"):
        N, c = 4, 16
        S = N * c
        for r in range(1, N):
            per_rank = {L.visible_pairs(layout, N, S, i, L.ring_source(i, r, N)) for i in range(N)}
            assert max(per_rank) - min(per_rank) <= (c if layout == "striped" else 0)
