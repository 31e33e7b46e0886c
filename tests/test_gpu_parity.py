"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (max abs error): bf16 inputs 2e-2 on O and 1e-3 on lse; fp32 inputs
1e-4 on O and 1e-5 on lse.  Token permutation and mask indexing are bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from oracle import layout as L
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64, positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _dev(*ts):
    return [t.cuda() for t in ts]


# ------------------------------------------------------------------ block attention

BLOCK_CASES = [
    # dtype, d, causal, sq, sk, hq, hkv, q positions, k positions (callables of sq/sk)
    ("bf16", 128, True, 128, 128, 2, 1, "diag"),
    ("bf16", 128, True, 300, 300, 4, 2, "diag"),        # ragged, several tiles
    ("bf16", 128, True, 1, 1, 1, 1, "diag"),
    ("bf16", 128, True, 129, 257, 2, 2, "later_q"),     # q after k: full tiles + ragged keys
    ("bf16", 128, True, 200, 200, 2, 1, "later_k"),     # k after q: every tile skipped
    ("bf16", 128, False, 190, 333, 8, 2, "diag"),
    ("bf16", 64, True, 256, 256, 4, 4, "diag"),
    ("bf16", 64, False, 77, 130, 2, 1, "diag"),
    ("bf16", 128, True, 384, 384, 2, 1, "zigzag"),      # 2 segments, tiles straddle them
    ("bf16", 128, True, 256, 256, 2, 1, "striped"),
    ("fp32", 64, True, 130, 130, 2, 2, "diag"),
    ("fp32", 128, False, 64, 100, 2, 1, "diag"),
    ("fp32", 64, True, 96, 96, 2, 1, "zigzag"),
]


def _block_ranges(kind, sq, sk):
    if kind == "diag":
        return ((0,), (sq,), 1), ((0,), (sk,), 1)
    if kind == "later_q":
        return ((sk,), (sq,), 1), ((0,), (sk,), 1)
    if kind == "later_k":
        return ((0,), (sq,), 1), ((sq + 5,), (sk,), 1)
    if kind == "zigzag":  # rank 1 of N=2 against rank 0
        S = 2 * sq
        from context_attention_cp_b200 import layout_range
        return layout_range("zigzag", 2, S, 1), layout_range("zigzag", 2, S, 0)
    if kind == "striped":  # rank 0 of N=4 against rank 2 (offset diagonal excluded)
        from context_attention_cp_b200 import layout_range
        return layout_range("striped", 4, 4 * sq, 0), layout_range("striped", 4, 4 * sk, 2)
    raise ValueError(kind)


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: "-".join(map(str, c)))
def test_block_attn_matches_oracle(cp, case):
    dt, d, causal, sq, sk, hq, hkv, kind = case
    q, _, _ = W.random_qkv(2, sq, hq, hkv, d, dt, seed=sq * 7 + sk)
    _, k, v = W.random_qkv(2, sk, hq, hkv, d, dt, seed=sq + 3 * sk)
    qr, kr = _block_ranges(kind, sq, sk)
    scale = d ** -0.5
    qd, kd, vd = _dev(q, k, v)
    o = torch.empty_like(qd)
    lse = torch.empty((2, hq, sq), dtype=torch.float32, device="cuda")
    cp.block_attn_fwd(qd, kd, vd, qr, kr, causal, scale, o, lse)
    cp.stream_check()
    ro, rl = oracle.attention(np64(q), np64(k), np64(v), causal, scale, pos_q=positions(qr), pos_k=positions(kr))
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l, "lse")
    assert_close_o(np64(o), ro, tol_o, "o")
    if kind == "later_k":
        assert torch.all(o == 0) and torch.all(lse == -math.inf)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_block_attn_fp32_output_and_accumulate(cp, dt):
    """accumulate=0 into fp32 o, then accumulate=1 of a second key block: the fused
    epilogue merge must equal attention over the union of the two key blocks."""
    b, sq, hq, hkv, d = 1, 200, 4, 2, 128
    q, k1, v1 = W.random_qkv(b, sq, hq, hkv, d, dt, seed=11)
    _, k2, v2 = W.random_qkv(b, 150, hq, hkv, d, dt, seed=12)
    qr = ((300,), (sq,), 1)
    kr1 = ((0,), (sq,), 1)
    kr2 = ((200,), (150,), 1)
    qd, k1d, v1d, k2d, v2d = _dev(q, k1, v1, k2, v2)
    o = torch.empty((b, sq, hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((b, hq, sq), dtype=torch.float32, device="cuda")
    cp.block_attn_fwd(qd, k1d, v1d, qr, kr1, True, d ** -0.5, o, lse)
    cp.block_attn_fwd(qd, k2d, v2d, qr, kr2, True, d ** -0.5, o, lse, accumulate=True)
    cp.stream_check()
    kk = np.concatenate([np64(k1), np64(k2)], axis=1)
    vv = np.concatenate([np64(v1), np64(v2)], axis=1)
    ro, rl = oracle.attention(np64(q), kk, vv, True, d ** -0.5, pos_q=positions(qr),
                              pos_k=np.concatenate([positions(kr1), positions(kr2)]))
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


# ------------------------------------------------------------------ merge

@pytest.mark.parametrize("ob_dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("out", [None, "bf16", "fp32"])
@pytest.mark.parametrize("d", [128, 64])
def test_lse_merge_matches_oracle(cp, ob_dtype, out, d):
    g = torch.Generator().manual_seed(5)
    b, s, h = 2, 37, 3
    o_acc = torch.randn((b, s, h, d), generator=g)
    o_b = torch.randn((b, s, h, d), generator=g).to(W.torch_dtype(ob_dtype))
    lse_acc = torch.randn((b, h, s), generator=g) * 10
    lse_b = torch.randn((b, h, s), generator=g) * 10
    lse_acc[0, 0, :5] = -math.inf
    lse_b[0, 0, 3:8] = -math.inf
    lse_b[1, 2, 10:12] = -math.inf
    ro, rl = oracle.lse_merge(np64(o_acc).transpose(0, 2, 1, 3), np64(lse_acc),
                              np64(o_b).transpose(0, 2, 1, 3), np64(lse_b))
    ro = ro.transpose(0, 2, 1, 3)
    oa, la, obd, lbd = _dev(o_acc, lse_acc, o_b, lse_b)
    o_out = None if out is None else torch.empty((b, s, h, d), dtype=W.torch_dtype(out), device="cuda")
    res, _ = cp.lse_merge(oa, la, obd, lbd, o_out)
    cp.stream_check()
    assert_close_lse(np64(la), rl, 1e-5)
    tol = 2e-2 if out == "bf16" else 1e-5
    assert_close_o(np64(res), ro, tol)
    if out is not None:
        assert torch.equal(oa.cpu(), o_acc)  # accumulator left untouched


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S", [(2, 512), (4, 8192), (8, 1024), (3, 96)])
def test_permute_is_bit_exact(cp, layout, N, S):
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zig-zag needs S % 2N == 0")
    g = torch.Generator().manual_seed(S + N)
    x = torch.randn((2, S, 3, 64), generator=g).to(torch.bfloat16)
    xd = x.cuda()
    xr = cp.layout_permute(xd, layout, N)
    want = L.permute(x.view(torch.int16).numpy(), layout, N, axis=1)
    assert np.array_equal(xr.cpu().view(torch.int16).numpy(), want)
    back = cp.layout_permute(xr, layout, N, inverse=True)
    assert torch.equal(back.cpu().view(torch.int16), x.view(torch.int16))
    lse = torch.randn((2, 5, S), generator=g)
    lr = cp.layout_permute(lse.cuda(), layout, N, seq_axis=2)
    assert np.array_equal(lr.cpu().view(torch.int32).numpy(),
                          L.permute(lse.view(torch.int32).numpy(), layout, N, axis=2))


@pytest.mark.parametrize("layout,N,S", [("zigzag", 4, 1024), ("striped", 3, 96), ("contiguous", 8, 1024)])
@pytest.mark.parametrize("H,d,dt", [(9, 128, "bf16"), (1, 37, "fp32"), (1, 33, "bf16"), (2, 160, "fp32"),
                                    (72, 130, "bf16")])
def test_permute_long_rows_bit_exact(cp, layout, N, S, H, d, dt):
    """Rows of at least 32 copy pieces (16-, 4- and 1-byte pieces, ragged passes);
    rows of 18720 bytes go in segments of 8 KB with a ragged last one."""
    g = torch.Generator().manual_seed(S + N + d)
    x = torch.randn((2, S, H, d), generator=g).to(W.torch_dtype(dt))
    bits = torch.int16 if dt == "bf16" else torch.int32
    xr = cp.layout_permute(x.cuda(), layout, N)
    assert np.array_equal(xr.cpu().view(bits).numpy(), L.permute(x.view(bits).numpy(), layout, N, axis=1))
    back = cp.layout_permute(xr, layout, N, inverse=True)
    assert torch.equal(back.cpu().view(bits), x.view(bits))


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S,H", [(4, 24, 5), (3, 18, 5), (8, 4096, 5), (2, 8, 5), (2, 16384, 5), (4, 65536, 40)])
def test_permute_lse_rows_bit_exact(cp, layout, N, S, H):
    """4-byte rows, sequence last, both directions: groups of 4 that straddle a
    zig-zag chunk or a rank (S = 24 over 4 ranks: chunks of 3), S % 4 != 0; rank
    chunks that hold whole 4096-row spans (S = 16384 over 2 ranks, and 65536 over 4
    with 3 x 40 rows: more spans than the grid has CTAs)."""
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zig-zag needs S % 2N == 0")
    g = torch.Generator().manual_seed(7 * S + N)
    lse = torch.randn((3, H, S), generator=g)
    want = L.permute(lse.view(torch.int32).numpy(), layout, N, axis=2)
    lr = cp.layout_permute(lse.cuda(), layout, N, seq_axis=2)
    assert np.array_equal(lr.cpu().view(torch.int32).numpy(), want)
    back = cp.layout_permute(lr, layout, N, seq_axis=2, inverse=True)
    assert torch.equal(back.cpu().view(torch.int32), lse.view(torch.int32))


# ------------------------------------------------------------------ ring

def _ring_on_gpu(cp, q, k, v, layout, N, causal, mode):
    qd, kd, vd = _dev(q, k, v)
    qr, kr, vr = (cp.layout_permute(t, layout, N) for t in (qd, kd, vd))
    o, lse = cp.ring_attn_fwd(qr, kr, vr, layout, N, causal, mode=mode)
    o = cp.layout_permute(o, layout, N, inverse=True)
    lse = cp.layout_permute(lse, layout, N, seq_axis=2, inverse=True)
    cp.stream_check()
    return o, lse


RING_CASES = [
    # layout, N, S, causal, hq, hkv, d, dtype
    ("contiguous", 2, 512, True, 4, 2, 128, "bf16"),
    ("zigzag", 4, 1024, True, 4, 1, 128, "bf16"),
    ("zigzag", 2, 768, True, 2, 2, 128, "bf16"),     # chunk 192: tiles straddle chunks
    ("striped", 4, 1024, True, 4, 2, 128, "bf16"),
    ("striped", 3, 600, True, 2, 1, 64, "bf16"),     # ragged c = 200
    ("contiguous", 4, 1024, False, 2, 2, 128, "bf16"),
    ("contiguous", 1, 320, True, 2, 1, 128, "bf16"),
    ("zigzag", 2, 512, True, 2, 1, 64, "fp32"),
    ("striped", 2, 256, True, 2, 2, 64, "fp32"),
]


@pytest.mark.parametrize("mode", ["fused", "stepwise", "stepwise_epi"])
@pytest.mark.parametrize("case", RING_CASES, ids=lambda c: "-".join(map(str, c)))
def test_ring_matches_oracle(cp, case, mode):
    layout, N, S, causal, hq, hkv, d, dt = case
    q, k, v = W.random_qkv(1, S, hq, hkv, d, dt, seed=S + N)
    o, lse = _ring_on_gpu(cp, q, k, v, layout, N, causal, mode)
    ro, rl = oracle.ring_attention(np64(q), np64(k), np64(v), layout, N, causal, d ** -0.5)
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


@pytest.mark.parametrize("mode", ["fused", "stepwise", "stepwise_epi"])
@pytest.mark.parametrize("layout,N,S", [("zigzag", 4, 1024), ("striped", 2, 512)])
def test_ring_batched_gqa_matches_oracle(cp, layout, N, S, mode):
    """Two batch entries and groups of four query heads per kv head, every output
    element: the kernel's grid runs (batch, kv head) outermost and the query heads of
    a group innermost, so every decoded (batch, kv head, rank, query head) must land
    on its own rows."""
    q, k, v = W.random_qkv(2, S, 8, 2, 128, "bf16", seed=S + 7 * N)
    o, lse = _ring_on_gpu(cp, q, k, v, layout, N, True, mode)
    ro, rl = oracle.ring_attention(np64(q), np64(k), np64(v), layout, N, True, 128 ** -0.5)
    tol_o, tol_l = TOL["bf16"]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


def test_fp32_workload_full(cp):
    """The fp32 S=256 contiguous N=2 workload, every output element."""
    w = W.BY_NAME["fp32_s256_contig2"]
    q, k, v = W.make_inputs(w)
    for mode in ("fused", "stepwise", "stepwise_epi"):
        o, lse = _ring_on_gpu(cp, q, k, v, w.layout, w.N, w.causal, mode)
        ro, rl = oracle.ring_attention(np64(q), np64(k), np64(v), w.layout, w.N, w.causal, w.scale)
        assert_close_lse(np64(lse), rl, 1e-5, mode)
        assert_close_o(np64(o), ro, 1e-4, mode)


# ------------------------------------------------------------------ mask counting

@pytest.mark.parametrize("layout,N,S", [("contiguous", 4, 512), ("zigzag", 4, 1024), ("striped", 4, 512),
                                        ("zigzag", 2, 768)])
def test_mask_counts_bit_exact_with_zero_queries(cp, layout, N, S):
    """Q = 0 makes every score 0, so exp(lse_b) is the number of visible keys of the
    row in that block: the device mask must agree with the oracle's integer
    enumeration for every row of every (rank, step) block."""
    c = S // N
    q, k, v = W.random_qkv(1, S, 2, 1, 128, "bf16", seed=3, q_zero=True)
    qd, kd, vd = _dev(q, k, v)
    qr_t, kr_t, vr_t = (cp.layout_permute(t, layout, N) for t in (qd, kd, vd))
    for i in range(N):
        pq = L.rank_positions(layout, N, S, i)
        for r in range(N):
            j = L.ring_source(i, r, N)
            pk = L.rank_positions(layout, N, S, j)
            o = torch.empty((1, c, 2, 128), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((1, 2, c), dtype=torch.float32, device="cuda")
            cp.block_attn_fwd(qr_t[:, i * c:(i + 1) * c], kr_t[:, j * c:(j + 1) * c], vr_t[:, j * c:(j + 1) * c],
                              cp.layout_range(layout, N, S, i), cp.layout_range(layout, N, S, j), True, 0.088,
                              o, lse)
            counts = np.rint(np.exp(np64(lse[0, 0]))).astype(np.int64)
            want = np.array([sum(1 for b_ in pk if b_ <= a) for a in pq])
            assert np.array_equal(counts, want), (i, j)
    o, lse = cp.ring_attn_fwd(qr_t, kr_t, vr_t, layout, N, True)
    lse = cp.layout_permute(lse, layout, N, seq_axis=2, inverse=True)
    counts = np.rint(np.exp(np64(lse[0, 1]))).astype(np.int64)
    assert np.array_equal(counts, np.arange(1, S + 1))


def test_ring_is_deterministic(cp):
    q, k, v = W.random_qkv(1, 2048, 8, 2, 128, "bf16", seed=9)
    o1, l1 = _ring_on_gpu(cp, q, k, v, "zigzag", 4, True, "fused")
    o2, l2 = _ring_on_gpu(cp, q, k, v, "zigzag", 4, True, "fused")
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_layouts_agree_after_unpermute(cp):
    """Permutation equivariance: the three layouts give the same attention."""
    q, k, v = W.random_qkv(1, 1024, 4, 2, 128, "bf16", seed=21)
    res = [_ring_on_gpu(cp, q, k, v, lay, 4, True, "fused") for lay in L.LAYOUTS]
    for o, lse in res[1:]:
        assert (o.float() - res[0][0].float()).abs().max().item() <= 2e-2
        assert (lse - res[0][1]).abs().max().item() <= 1e-3
