"""The effective-FLOP count the benchmark divides by, pinned to the ring's schedule.

"上下文并行与 Ring Attention" (hs-black.github.io), section 能否把通信藏住: one ring
step of a rank costs T_math = 4 b c^2 h / C, i.e. 4 multiply-add flops per
(query, key) pair and head dimension (QK^T and PV).  Summed over every rank and
every ring step (the schedule of section Ring Attention, source (i - r) mod N) the
visible pairs are those of the whole sequence under the mask, so the effective
FLOPs of a workload are 4 * b * Hq * d * pairs with pairs = S(S+1)/2 causal and S^2
without the mask (per document under a document mask).  These tests count the pairs
step by step with the oracle's position maps and compare."""
import itertools

import pytest

import cp_workloads as W
from oracle import layout as L


def _pairs_by_schedule(layout, N, S, causal, doc_starts):
    """Visible (query, key) pairs summed over ranks i and steps r, each step pairing
    rank i's queries with the keys of rank (i - r) mod N."""
    bounds = doc_starts + [S]
    doc = {}
    for a, e in zip(bounds[:-1], bounds[1:]):
        for p in range(a, e):
            doc[p] = a
    total = 0
    for i in range(N):
        pq = L.rank_positions(layout, N, S, i)
        for r in range(N):
            pk = L.rank_positions(layout, N, S, L.ring_source(i, r, N))
            total += sum(1 for p, t in itertools.product(pq, pk) if doc[p] == doc[t] and ((not causal) or t <= p))
    return total


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S", [(1, 16), (2, 32), (4, 64), (3, 48)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n_docs", [1, 5])
def test_visible_pairs_equal_the_schedule_count(layout, N, S, causal, n_docs):
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zig-zag needs S % 2N == 0")
    w = W.Workload(name="t", index=3, dtype="bf16", b=2, hq=4, hkv=2, d=8, S=S, causal=causal, layout=layout, N=N,
                   n_docs=n_docs)
    starts = w.doc_starts()
    assert len(starts) == n_docs
    assert w.visible_pairs() == _pairs_by_schedule(layout, N, S, causal, starts)
    assert w.effective_flops() == 4 * w.b * w.hq * w.d * w.visible_pairs()


def test_named_workloads_closed_forms():
    """Every named workload: S(S+1)/2 pairs causal, S^2 without the mask (one
    document), and the non-causal total equals N^2 full c x c steps of the page's
    T_math; the headline workload's count, 2.815e14 effective FLOPs, is the one the
    bench's TFLOP/s rests on."""
    for w in W.WORKLOADS:
        if w.n_docs > 1:
            continue
        want = w.S * (w.S + 1) // 2 if w.causal else w.S * w.S
        assert w.visible_pairs() == want, w.name
        if not w.causal:
            assert w.effective_flops() == w.N ** 2 * 4 * w.b * w.c ** 2 * w.hq * w.d, w.name
    head = W.BY_NAME[W.BENCH_WORKLOAD]
    assert head.name == "llama3_70b_s128k_zigzag8"
    assert head.effective_flops() == 4 * 1 * 64 * 128 * (131072 * 131073 // 2)
    assert round(head.effective_flops() / 1e14, 3) == 2.815
