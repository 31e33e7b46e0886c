"""GPU parity of All-Gather context parallelism (cp_allgather_attn_fwd through the C
ABI) against the fp64 oracle, with and without the document mask (section
All-Gather 式 CP).  Tolerances as for the ring: bf16 2e-2 on O, 1e-3 on lse.
"""
import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _allgather(cp, q, k, v, layout, N, causal, docs):
    qr, kr, vr = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v))
    o, lse = cp.allgather_attn_fwd(qr, kr, vr, layout, N, causal, docs)
    o = cp.layout_permute(o, layout, N, inverse=True)
    lse = cp.layout_permute(lse, layout, N, seq_axis=2, inverse=True)
    cp.stream_check()
    return o, lse


# More document starts than one launch of the table kernel takes (2048 per launch):
# 2500 documents of a few tokens each over 8192 positions.
MANY_DOCS = [0] + sorted(int(x) for x in np.random.default_rng(5).choice(np.arange(1, 8192), 2499, replace=False))

CASES = [
    # layout, N, S, b, hq, hkv, document starts
    ("zigzag", 4, 1024, 1, 4, 2, [0, 100, 101, 400, 777]),
    ("zigzag", 2, 424, 2, 2, 2, [0, 5, 211, 212, 300]),       # c = 212, starts inside tiles and chunks
    ("striped", 4, 1024, 1, 4, 1, [0, 128, 255, 256, 1000]),
    ("contiguous", 3, 390, 1, 2, 1, [0, 129, 130, 389]),      # a one-token document at the end
    ("contiguous", 1, 640, 1, 2, 2, [0, 64, 320]),
    ("zigzag", 8, 2048, 1, 8, 2, list(range(0, 2048, 97))),   # many short documents
    ("zigzag", 4, 1024, 1, 4, 2, [0]),                        # no mask: plain causal attention
    ("zigzag", 4, 8192, 1, 2, 1, MANY_DOCS),                  # two launches of the table kernel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c[:6]) + "-d%d" % len(c[6]))
def test_allgather_matches_oracle(cp, case):
    layout, N, S, b, hq, hkv, docs = case
    q, k, v = W.random_qkv(b, S, hq, hkv, 128, "bf16", seed=S + N + len(docs))
    o, lse = _allgather(cp, q, k, v, layout, N, True, docs)
    ro, rl = oracle.allgather_attention(np64(q), np64(k), np64(v), layout, N, True, 128 ** -0.5, docs)
    tol_o, tol_l = TOL["bf16"]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


OTHER_CASES = [
    # layout, N, S, b, hq, hkv, d, dtype, document starts: the FFMA kernels (fp32) and
    # the tensor-core kernel's d = 64 instantiation
    ("zigzag", 4, 512, 1, 4, 2, 64, "fp32", [0, 100, 101, 400]),
    ("striped", 2, 260, 2, 2, 1, 128, "fp32", [0, 7, 130]),
    ("contiguous", 3, 390, 1, 2, 2, 64, "fp32", [0]),
    ("zigzag", 2, 424, 1, 4, 2, 64, "bf16", [0, 5, 211, 212, 300]),
]


@pytest.mark.parametrize("case", OTHER_CASES, ids=lambda c: "-".join(str(x) for x in c[:8]) + "-d%d" % len(c[8]))
def test_allgather_fp32_and_d64_match_oracle(cp, case):
    layout, N, S, b, hq, hkv, d, dt, docs = case
    q, k, v = W.random_qkv(b, S, hq, hkv, d, dt, seed=S + N + d)
    o, lse = _allgather(cp, q, k, v, layout, N, True, docs)
    assert o.dtype == q.dtype
    ro, rl = oracle.allgather_attention(np64(q), np64(k), np64(v), layout, N, True, d ** -0.5, docs)
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


def test_allgather_without_documents_matches_ring(cp):
    q, k, v = W.random_qkv(1, 2048, 8, 2, 128, "bf16", seed=5)
    o1, l1 = _allgather(cp, q, k, v, "zigzag", 4, True, None)
    qr, kr, vr = (cp.layout_permute(t.cuda(), "zigzag", 4) for t in (q, k, v))
    o2, l2 = cp.ring_attn_fwd(qr, kr, vr, "zigzag", 4, True)
    o2 = cp.layout_permute(o2, "zigzag", 4, inverse=True)
    l2 = cp.layout_permute(l2, "zigzag", 4, seq_axis=2, inverse=True)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_document_mask_counts_bit_exact(cp):
    """Q = 0: every visible score is 0, so exp(lse) counts the visible keys of a row:
    pos - (its document start) + 1 with the causal document mask."""
    S, N = 1024, 4
    docs = [0, 3, 130, 131, 500, 1023]
    q, k, v = W.random_qkv(1, S, 2, 1, 128, "bf16", seed=8, q_zero=True)
    _, lse = _allgather(cp, q, k, v, "zigzag", N, True, docs)
    counts = np.rint(np.exp(np64(lse[0, 0]))).astype(np.int64)
    starts = np.array(docs)
    want = np.array([p - starts[np.searchsorted(starts, p, side="right") - 1] + 1 for p in range(S)])
    assert np.array_equal(counts, want)


def test_allgather_argument_errors(cp):
    q, k, v = (t.cuda() for t in W.random_qkv(1, 256, 4, 2, 128, "bf16", seed=1))
    for docs in ([1, 10], [0, 10, 10], [0, 300]):
        with pytest.raises(cp.CPError) as e:
            cp.allgather_attn_fwd(q, k, v, "zigzag", 2, True, docs)
        assert e.value.code == 1
    with pytest.raises(cp.CPError) as e:
        cp.allgather_attn_fwd(q, k, v, "zigzag", 2, False, [0, 100])
    assert e.value.code == 2
    q256 = torch.zeros((1, 256, 4, 256), dtype=torch.bfloat16, device="cuda")
    k256 = torch.zeros((1, 256, 2, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cp.CPError) as e:
        cp.allgather_attn_fwd(q256, k256, k256, "zigzag", 2, True, None)   # head dim 256
    assert e.value.code == 2


def test_full_size_documents_sampled(cp):
    """The 8-document 8B workload at full size, the launch the bench times."""
    from gpu_helpers import sample_rows
    w = W.BY_NAME["llama3_8b_s8k_zigzag4_docs8"]
    q, k, v = W.make_inputs(w)
    docs = w.doc_starts()
    o, lse = _allgather(cp, q, k, v, w.layout, w.N, w.causal, docs)
    sel = sample_rows(w, n_random=24, seed=w.seed)
    extra = []
    for n, s0 in enumerate(docs):  # each document's first row and the row before it
        extra.append((0, (3 * n) % w.hq, s0))
        if s0 > 0:
            extra.append((0, (3 * n + 1) % w.hq, s0 - 1))
    sel = np.concatenate([sel, np.array(extra, dtype=np.int64)])
    q_sel = np.stack([np64(q[b, p, h]) for b, h, p in sel])
    ro, rl = oracle.attention_rows_doc(q_sel, sel, np64(k), np64(v), w.causal, w.scale, w.hq, docs)
    got_o = np.stack([np64(o[b, p, h]) for b, h, p in sel])
    got_l = np.array([float(lse[b, h, p]) for b, h, p in sel])
    tol_o, tol_l = TOL["bf16"]
    assert_close_lse(got_l, rl, tol_l)
    assert_close_o(got_o, ro, tol_o)


# ------------------------------------------------------------------ backward

BWD_CASES = [
    ("zigzag", 4, 1024, 1, 4, 2, [0, 100, 101, 400, 777]),
    ("zigzag", 2, 424, 2, 2, 2, [0, 5, 211, 212, 300]),
    ("striped", 4, 1024, 1, 4, 1, [0, 128, 255, 256, 1000]),
    ("contiguous", 3, 390, 1, 2, 1, [0, 129, 130, 389]),
    ("zigzag", 8, 2048, 1, 8, 2, list(range(0, 2048, 97))),
    ("zigzag", 4, 1024, 1, 4, 2, [0]),
    ("zigzag", 4, 8192, 1, 2, 1, MANY_DOCS),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "-".join(str(x) for x in c[:6]) + "-d%d" % len(c[6]))
def test_allgather_bwd_matches_oracle(cp, case):
    layout, N, S, b, hq, hkv, docs = case
    d = 128
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "bf16", seed=2 * S + N)
    do = W.random_do(b, S, hq, d, "bf16", seed=2 * S + N)
    qr, kr, vr, dor = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v, do))
    o, lse = cp.allgather_attn_fwd(qr, kr, vr, layout, N, True, docs)
    grads = cp.allgather_attn_bwd(qr, kr, vr, o, lse, dor, layout, N, True, docs)
    grads = [cp.layout_permute(g, layout, N, inverse=True) for g in grads]
    cp.stream_check()
    want = oracle.allgather_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, True, d ** -0.5, docs)
    for name, g, w in zip(("dq", "dk", "dv"), grads, want):
        err = np.max(np.abs(np64(g) - w))
        assert err <= 2e-2 * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))


@pytest.mark.parametrize("case", OTHER_CASES, ids=lambda c: "-".join(str(x) for x in c[:8]) + "-d%d" % len(c[8]))
def test_allgather_bwd_fp32_and_d64_match_oracle(cp, case):
    """The FFMA backward in its All-Gather form (one gathered key block, documents):
    fp32 within 1e-4 x max |reference|, bf16 within 2e-2 x max |reference|."""
    layout, N, S, b, hq, hkv, d, dt, docs = case
    q, k, v = W.random_qkv(b, S, hq, hkv, d, dt, seed=3 * S + N + d)
    do = W.random_do(b, S, hq, d, dt, seed=3 * S + N + d)
    qr, kr, vr, dor = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v, do))
    o, lse = cp.allgather_attn_fwd(qr, kr, vr, layout, N, True, docs)
    grads = cp.allgather_attn_bwd(qr, kr, vr, o, lse, dor, layout, N, True, docs)
    grads = [cp.layout_permute(g, layout, N, inverse=True) for g in grads]
    cp.stream_check()
    want = oracle.allgather_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, True, d ** -0.5, docs)
    tol = 1e-4 if dt == "fp32" else 2e-2
    for name, g, w in zip(("dq", "dk", "dv"), grads, want):
        assert g.dtype == q.dtype
        err = np.max(np.abs(np64(g) - w))
        assert err <= tol * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))
