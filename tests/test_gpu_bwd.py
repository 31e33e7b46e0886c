"""GPU parity of the ring backward (cp_ring_attn_bwd through the C ABI) against the
fp64 oracle's gradients (section 分块注意力, paragraph on the backward pass).

Tolerance, from the arithmetic of the bf16 path: Q, K, V, dO enter exactly; P and
dS are rounded to bf16 before the tensor-core products (relative error u = 2^-8
at most each), products accumulate in fp32, D = dO . o uses the forward's bf16 o,
and the results are rounded to bf16 once more (u / 2).  Each gradient element is
a sum whose terms carry a relative error of at most about 2u, so the error is
bounded by a small multiple of u times the size of the summands; against the
largest reference element that gives the bar used here,
    max |got - ref| <= 2e-2 * max |ref|     (per gradient tensor),
about five bf16 ulps of the largest element.  dK and dV are summed in a fixed
order and must be bit-identical across runs; dQ sums with atomic reductions.
"""
import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import np64, positions

pytestmark = pytest.mark.gpu

TOL_REL = 2e-2


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _fwd_bwd(cp, q, k, v, do, layout, N, causal, scale):
    """Original-order CPU inputs -> rank-major device tensors -> ring forward and
    backward -> gradients back in original order (device tensors)."""
    qr, kr, vr, dor = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v, do))
    o, lse = cp.ring_attn_fwd(qr, kr, vr, layout, N, causal, scale)
    dq, dk, dv = cp.ring_attn_bwd(qr, kr, vr, o, lse, dor, layout, N, causal, scale)
    cp.stream_check()
    return tuple(cp.layout_permute(t, layout, N, inverse=True) for t in (dq, dk, dv))


def _assert_grad(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    ref = np.max(np.abs(want)) if want.size else 0.0
    err = np.max(np.abs(got - want)) if want.size else 0.0
    assert err <= TOL_REL * ref, "%s: max abs err %.3g > %.3g (max |ref| %.3g)" % (what, err, TOL_REL * ref, ref)
    return err / ref if ref else 0.0


BWD_CASES = [
    # layout, N, S, causal, b, hq, hkv
    ("contiguous", 2, 512, True, 1, 4, 2),
    ("zigzag", 4, 1024, True, 1, 4, 1),
    ("zigzag", 2, 424, True, 2, 2, 2),       # c = 212: ragged query and key tiles
    ("striped", 4, 1024, True, 1, 4, 2),
    ("striped", 3, 390, True, 1, 2, 1),      # c = 130: a key tile of two keys
    ("contiguous", 4, 1024, False, 1, 2, 2),
    ("contiguous", 1, 320, True, 2, 2, 1),
    ("contiguous", 3, 96, True, 1, 2, 2),    # c = 32, less than one query tile
    ("zigzag", 8, 2048, True, 1, 8, 2),
    ("zigzag", 4, 1024, True, 2, 8, 2),      # two batch entries, groups of four query heads
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "-".join(map(str, c)))
def test_ring_bwd_matches_oracle(cp, case):
    layout, N, S, causal, b, hq, hkv = case
    d = 128
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "bf16", seed=S + 3 * N)
    do = W.random_do(b, S, hq, d, "bf16", seed=S + 3 * N)
    dq, dk, dv = _fwd_bwd(cp, q, k, v, do, layout, N, causal, d ** -0.5)
    want = oracle.ring_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, causal, d ** -0.5)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        _assert_grad(np64(g), w, name)


# The FFMA backward: fp32 inputs (d 64 and 128) and bf16 with d = 64.  fp32 bar: the
# forward's o and lse enter with at most 1e-4 / 1e-5 absolute error (the forward's
# fp32 bar), which reaches p = e^{x - lse} and D = dO . o as relative errors of that
# size; every product and sum is fp32 (unit roundoff 2^-24, at most S terms per
# sum).  So  max |got - ref| <= 1e-4 * max |ref|  per gradient tensor.  bf16 with
# d = 64 computes in fp32 and rounds once to bf16: the bf16 bar above.
TOL_REL_FP32 = 1e-4

FFMA_CASES = [
    # layout, N, S, causal, b, hq, hkv, d, dtype
    ("contiguous", 2, 256, True, 1, 2, 2, 64, "fp32"),
    ("zigzag", 4, 512, True, 2, 4, 2, 128, "fp32"),
    ("striped", 3, 390, True, 1, 4, 1, 64, "fp32"),     # c = 130: ragged tiles
    ("contiguous", 2, 256, False, 1, 2, 2, 64, "fp32"),
    ("zigzag", 2, 424, True, 1, 4, 2, 64, "bf16"),
    ("contiguous", 1, 200, True, 1, 2, 1, 64, "bf16"),
]


@pytest.mark.parametrize("case", FFMA_CASES, ids=lambda c: "-".join(map(str, c)))
def test_ring_bwd_ffma_matches_oracle(cp, case):
    layout, N, S, causal, b, hq, hkv, d, dt = case
    q, k, v = W.random_qkv(b, S, hq, hkv, d, dt, seed=S + 7 * N + d)
    do = W.random_do(b, S, hq, d, dt, seed=S + 7 * N + d)
    dq, dk, dv = _fwd_bwd(cp, q, k, v, do, layout, N, causal, d ** -0.5)
    want = oracle.ring_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, causal, d ** -0.5)
    tol = TOL_REL_FP32 if dt == "fp32" else TOL_REL
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        assert g.dtype == q.dtype
        err = np.max(np.abs(np64(g) - w))
        assert err <= tol * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))


def test_fp32_workload_bwd_element_by_element(cp):
    """The fp32 workload (S = 256, contiguous N = 2, d = 64) at its full size."""
    w = W.BY_NAME["fp32_s256_contig2"]
    q, k, v = W.make_inputs(w)
    do = W.make_do(w)
    dq, dk, dv = _fwd_bwd(cp, q, k, v, do, w.layout, w.N, w.causal, w.scale)
    want = oracle.ring_attention_bwd(np64(q), np64(k), np64(v), np64(do), w.layout, w.N, w.causal, w.scale)
    for name, g, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        err = np.max(np.abs(np64(g) - ref))
        assert err <= TOL_REL_FP32 * np.max(np.abs(ref)), (name, err)


@pytest.mark.parametrize("dt,d,kind", [("bf16", 128, "zigzag"), ("fp32", 64, "zigzag"), ("bf16", 64, "striped"),
                                       ("fp32", 128, "later_q"), ("bf16", 128, "striped"), ("bf16", 128, "later_q"),
                                       ("bf16", 128, "contiguous")])
def test_block_bwd_adds_the_block_share(cp, dt, d, kind):
    """cp_block_attn_bwd: one query block against one key block with the rows' global
    statistics; the shares are ADDED to fp32 accumulators (pre-filled here).  bf16
    with d = 128 runs the tensor-core kernel (the tensor-core backward's bar), the
    rest the FFMA kernels (the fp32 bar)."""
    from context_attention_cp_b200 import layout_range
    S, N = 512, 2
    q, k, v = W.random_qkv(1, S, 4, 2, d, dt, seed=S + d)
    do = W.random_do(1, S, 4, d, dt, seed=S + d)
    o_full, lse_full = oracle.attention(np64(q), np64(k), np64(v), True, d ** -0.5)
    if kind == "later_q":   # query block after the key block: every pair visible
        qr, kr = ((256,), (256,), 1), ((0,), (256,), 1)
    else:
        qr, kr = layout_range(kind, N, S, 1), layout_range(kind, N, S, 0)
    pq, pk = positions(qr), positions(kr)
    qi, ki = torch.from_numpy(pq), torch.from_numpy(pk)
    qb, kb, vb, dob = (t[:, idx].contiguous() for t, idx in ((q, qi), (k, ki), (v, ki), (do, qi)))
    ob = torch.from_numpy(o_full[:, pq]).to(q.dtype)   # the global forward's o of these rows
    lb = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, pq])).float()
    pre = 0.25
    acc = [torch.full(t.shape, pre, dtype=torch.float32, device="cuda") for t in (qb, kb, vb)]
    cp.block_attn_bwd(*(t.cuda() for t in (qb, kb, vb, ob, lb, dob)), qr, kr, True, d ** -0.5, *acc)
    cp.stream_check()
    delta = np.einsum("bshd,bshd->bhs", np64(dob), np64(ob))
    want = oracle.attention_bwd(np64(qb), np64(kb), np64(vb), np64(dob), True, d ** -0.5, pos_q=pq, pos_k=pk,
                                lse=np64(lb), delta=delta)[:3]
    rel = TOL_REL if (dt == "bf16" and d == 128) else 1e-4
    for name, g, w in zip(("dq", "dk", "dv"), acc, want):
        err = np.max(np.abs(np64(g) - pre - w))
        assert err <= rel * max(np.max(np.abs(w)), 1e-30) + 1e-6, (name, err, np.max(np.abs(w)))


@pytest.mark.parametrize("causal", [True, False])
def test_block_bwd_tensor_cores_two_blocks_ragged(cp, causal):
    """The tensor-core block backward called twice into the same accumulators, once
    per key block (the two steps a rank of a two-rank ring runs), with ragged query
    and key blocks (212 and 130 rows: partial tiles in both axes), b = 2 and GQA 4:1;
    the sums equal the oracle's gradients of the query block against both blocks."""
    from context_attention_cp_b200 import layout_range
    b, hq, hkv, d = 2, 8, 2, 128
    S = 212 + 130 + 130
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "bf16", seed=91)
    do = W.random_do(b, S, hq, d, "bf16", seed=91)
    o_full, lse_full = oracle.attention(np64(q), np64(k), np64(v), causal, d ** -0.5)
    qr = ((260,), (212,), 1)                      # query rows: positions 260 .. 471
    kr0, kr1 = ((0,), (130,), 1), ((130,), (130,), 1)
    pq, pk0, pk1 = positions(qr), positions(kr0), positions(kr1)
    qi = torch.from_numpy(pq)
    qb, dob = (t[:, qi].contiguous() for t in (q, do))
    ob = torch.from_numpy(o_full[:, pq]).to(torch.bfloat16)
    lb = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, pq])).float()
    dq_acc = torch.zeros(qb.shape, dtype=torch.float32, device="cuda")
    dks, dvs = [], []
    for kr, pk in ((kr0, pk0), (kr1, pk1)):
        ki = torch.from_numpy(pk)
        kb, vb = (t[:, ki].contiguous() for t in (k, v))
        dk_acc = torch.zeros(kb.shape, dtype=torch.float32, device="cuda")
        dv_acc = torch.zeros(kb.shape, dtype=torch.float32, device="cuda")
        cp.block_attn_bwd(*(t.cuda() for t in (qb, kb, vb, ob, lb, dob)), qr, kr, causal, None, dq_acc, dk_acc,
                          dv_acc)
        dks.append(dk_acc)
        dvs.append(dv_acc)
    cp.stream_check()
    delta = np.einsum("bshd,bshd->bhs", np64(dob), np64(ob))
    pk = np.concatenate([pk0, pk1])
    want = oracle.attention_bwd(np64(qb), np64(k[:, :260]), np64(v[:, :260]), np64(dob), causal, d ** -0.5,
                                pos_q=pq, pos_k=pk, lse=np64(lb), delta=delta)[:3]
    got = [dq_acc, torch.cat(dks, dim=1), torch.cat(dvs, dim=1)]
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        err = np.max(np.abs(np64(g) - w))
        assert err <= TOL_REL * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))


def test_ring_bwd_dkdv_deterministic(cp):
    q, k, v = W.random_qkv(1, 2048, 8, 2, 128, "bf16", seed=77)
    do = W.random_do(1, 2048, 8, 128, "bf16", seed=77)
    a = _fwd_bwd(cp, q, k, v, do, "zigzag", 4, True, 128 ** -0.5)
    b_ = _fwd_bwd(cp, q, k, v, do, "zigzag", 4, True, 128 ** -0.5)
    assert torch.equal(a[1].view(torch.int16), b_[1].view(torch.int16))
    assert torch.equal(a[2].view(torch.int16), b_[2].view(torch.int16))
    assert (a[0].float() - b_[0].float()).abs().max().item() <= TOL_REL * a[0].float().abs().max().item()


def test_ring_bwd_layouts_agree(cp):
    """Permutation equivariance: the three layouts give the same gradients."""
    q, k, v = W.random_qkv(1, 1024, 4, 2, 128, "bf16", seed=31)
    do = W.random_do(1, 1024, 4, 128, "bf16", seed=31)
    res = [_fwd_bwd(cp, q, k, v, do, lay, 4, True, 128 ** -0.5) for lay in ("contiguous", "zigzag", "striped")]
    for r in res[1:]:
        for g, g0 in zip(r, res[0]):
            assert (g.float() - g0.float()).abs().max().item() <= TOL_REL * g0.float().abs().max().item()


def test_ring_bwd_argument_errors(cp):
    q, k, v = (t.cuda() for t in W.random_qkv(1, 256, 4, 2, 128, "bf16", seed=1))
    o = torch.empty_like(q)
    lse = torch.empty((1, 4, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(cp.CPError) as e:
        cp.ring_attn_bwd(q, k, v, o, lse, q, "zigzag", 3, True)
    assert e.value.code == 3
    q256 = torch.zeros((1, 256, 4, 256), dtype=torch.bfloat16, device="cuda")
    k256 = torch.zeros((1, 256, 2, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cp.CPError) as e:
        cp.ring_attn_bwd(q256, k256, k256, q256, lse, q256, "zigzag", 2, True)   # head dim 256
    assert e.value.code == 2
    with pytest.raises(cp.CPError):
        cp.ring_attn_bwd(q, k, v, o, lse[:, :, :128], q, "zigzag", 2, True)


# ------------------------------------------------------------------ full sizes

def _key_samples(w, rng):
    """(batch, kv head, original key position): the last keys of the sequence, whose
    gradients the oracle reaches through few query rows, plus early keys when the
    sequence is short enough for the oracle to walk every query row."""
    pos = {w.S - 1, w.S - 2, w.S - 64, w.S - 129}
    pos.update(int(x) for x in rng.integers(w.S - 256, w.S, 4))
    if w.S <= 8192:
        pos.update({0, 1, 127, 128, w.S // 2, w.S // 4 - 1})
    sel = []
    for n, p in enumerate(sorted(pos)):
        sel.append((n % w.b, (5 * n) % w.hkv, p))
    return np.array(sel, dtype=np.int64)


def _query_samples(w, rng):
    pos = {0, 1, w.S - 1, w.S // 2, w.S // w.N, w.S // w.N - 1}
    pos.update(int(x) for x in rng.integers(0, w.S, 8))
    sel = []
    for n, p in enumerate(sorted(pos)):
        sel.append((n % w.b, (7 * n) % w.hq, p))
    return np.array(sel, dtype=np.int64)


BF16_WORKLOADS = [w.name for w in W.WORKLOADS if w.dtype == "bf16" and w.n_docs == 1]


@pytest.mark.parametrize("name", BF16_WORKLOADS)
def test_full_size_bwd_sampled(cp, name):
    """Every bf16 workload at full size through the same launch as the bench:
    sampled dq rows and dk, dv rows against the oracle, plus the row-sum identities
    sum_j dk_j = 0 and sum_j dv_j = sum of dO over the group's rows."""
    w = W.BY_NAME[name]
    q, k, v = W.make_inputs(w)
    do = W.make_do(w)
    dq, dk, dv = _fwd_bwd(cp, q, k, v, do, w.layout, w.N, w.causal, w.scale)
    rng = np.random.default_rng(w.seed)
    sel_q = _query_samples(w, rng)
    sel_k = _key_samples(w, rng) if w.causal else np.zeros((0, 3), np.int64)
    # the oracle sees only the query rows it needs: the sampled ones and (causal)
    # every row at or after the first sampled key
    need = set(int(x) for x in sel_q[:, 2])
    if len(sel_k):
        need.update(range(int(sel_k[:, 2].min()), w.S))
    rows = np.array(sorted(need), dtype=np.int64)
    where = {int(r): n for n, r in enumerate(rows)}
    sq = sel_q.copy()
    sq[:, 2] = [where[int(x)] for x in sel_q[:, 2]]
    ridx = torch.from_numpy(rows)
    gq, gk, gv = oracle.attention_bwd_sel(np64(q[:, ridx]), np64(k), np64(v), np64(do[:, ridx]), w.causal, w.scale,
                                          sq, sel_k, pos_q=rows)
    got_q = np.stack([np64(dq[b_, p, h]) for b_, h, p in sel_q])
    _assert_grad(got_q, gq, name + " dq")
    if len(sel_k):
        got_k = np.stack([np64(dk[b_, p, h]) for b_, h, p in sel_k])
        got_v = np.stack([np64(dv[b_, p, h]) for b_, h, p in sel_k])
        _assert_grad(got_k, gk, name + " dk")
        _assert_grad(got_v, gv, name + " dv")
    # identities at every size: the probabilities of a row sum to one
    u = 2.0 ** -8
    dk64, dv64 = dk.double(), dv.double()
    assert torch.all(dk64.sum(1).abs() <= u * dk64.abs().sum(1) + 1e-30)
    g = w.hq // w.hkv
    do_sum = do.cuda().double().sum(1).view(w.b, w.hkv, g, w.d).sum(2)
    assert torch.all((dv64.sum(1) - do_sum).abs() <= 2 * u * dv64.abs().sum(1))


@pytest.mark.parametrize("layout,hkv", [("striped", 1), ("zigzag", 1), ("contiguous", 1), ("striped", 2)])
def test_block_bwd_tensor_cores_every_ring_pair(cp, layout, hkv):
    """The tensor-core block backward for every (query rank, key rank) pair of a
    four-rank ring (the blocks a real rank meets: the diagonal block, blocks seen in
    full, strictly masked blocks, empty ones), GQA 4:1, against the oracle's shares
    of each pair with the global statistics."""
    from context_attention_cp_b200 import layout_range
    S, N, hq, d = 1024, 4, 4, 128
    q, k, v = W.random_qkv(1, S, hq, hkv, d, "bf16", seed=71)
    do = W.random_do(1, S, hq, d, "bf16", seed=71)
    o_full, lse_full = oracle.attention(np64(q), np64(k), np64(v), True, d ** -0.5)
    worst = []
    for i in range(N):
        qr = layout_range(layout, N, S, i)
        pq = positions(qr)
        qi = torch.from_numpy(pq)
        qb, dob = (t[:, qi].contiguous() for t in (q, do))
        ob = torch.from_numpy(o_full[:, pq]).to(torch.bfloat16)
        lb = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, pq])).float()
        delta = np.einsum("bshd,bshd->bhs", np64(dob), np64(ob))
        for j in range(N):
            kr = layout_range(layout, N, S, j)
            pk = positions(kr)
            ki = torch.from_numpy(pk)
            kb, vb = (t[:, ki].contiguous() for t in (k, v))
            acc = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in (qb, kb, vb)]
            cp.block_attn_bwd(*(t.cuda() for t in (qb, kb, vb, ob, lb, dob)), qr, kr, True, None, *acc)
            cp.stream_check()
            want = oracle.attention_bwd(np64(qb), np64(kb), np64(vb), np64(dob), True, d ** -0.5, pos_q=pq,
                                        pos_k=pk, lse=np64(lb), delta=delta)[:3]
            for name, g, w in zip(("dq", "dk", "dv"), acc, want):
                err = float(np.max(np.abs(np64(g) - w)))
                scale_ = float(np.max(np.abs(w)))
                worst.append((err - TOL_REL * scale_ - 1e-6, (i, j, name, err, scale_)))
    bad = [x for e, x in worst if e > 0]
    assert not bad, bad
