"""GPU parity of USP, Ulysses inside each ring group and the ring across groups
(cp_usp_attn_fwd / cp_usp_attn_bwd through the C ABI), against the fp64 oracle:
the exchange bit for bit against the oracle's index map, the attention within the
ring's tolerances (bf16 2e-2 on O and 1e-3 on lse; fp32 1e-4 and 1e-5), the
gradients within the backward's bar (2e-2 x max |reference| per tensor)."""
import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("layout,N,P,b,S,H", [("zigzag", 2, 2, 2, 64, 8), ("striped", 3, 2, 1, 96, 4),
                                              ("contiguous", 2, 4, 1, 128, 8), ("zigzag", 4, 2, 1, 8192, 32)])
def test_usp_exchange_is_bit_exact(cp, layout, N, P, b, S, H):
    """Rank-major input (the ring layout over N) through the Ulysses exchange with P:
    entry u, rows [g c, (g+1) c) must hold the oracle's rank (g, u) buffer."""
    d = 128
    x = torch.randn((b, S, H, d), generator=torch.Generator().manual_seed(S + N + P)).to(torch.bfloat16)
    xr = cp.layout_permute(x.cuda(), layout, N)
    y = cp.ulysses_all_to_all(xr, P)
    got = y.cpu().view(torch.int16).numpy().reshape(P, b, S, H // P, d)
    ref = oracle.usp_exchange(x.view(torch.int16).numpy(), layout, N, P)
    c = S // N
    for (g, u), blk in ref.items():
        assert np.array_equal(got[u, :, g * c:(g + 1) * c], blk), (g, u)
    back = cp.ulysses_all_to_all(y, P, inverse=True)
    assert torch.equal(back.view(torch.int16), xr.view(torch.int16))


def _usp(cp, q, k, v, layout, N, P, causal):
    qr, kr, vr = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v))
    o, lse = cp.usp_attn_fwd(qr, kr, vr, layout, N, P, causal)
    o = cp.layout_permute(o, layout, N, inverse=True)
    lse = cp.layout_permute(lse, layout, N, seq_axis=2, inverse=True)
    cp.stream_check()
    return o, lse


CASES = [
    # layout, N, P, b, S, hq, hkv, d, causal, dtype
    ("zigzag", 2, 2, 1, 1024, 8, 4, 128, True, "bf16"),
    ("striped", 4, 2, 1, 1024, 8, 2, 128, True, "bf16"),
    ("contiguous", 3, 2, 2, 600, 4, 2, 128, True, "bf16"),    # c = 200: ragged tiles
    ("zigzag", 2, 4, 1, 512, 8, 8, 64, False, "bf16"),
    ("zigzag", 4, 1, 1, 1024, 4, 2, 128, True, "bf16"),       # P = 1: the fused ring
    ("contiguous", 1, 4, 1, 512, 8, 4, 128, True, "bf16"),    # N = 1: Ulysses
    ("zigzag", 2, 2, 1, 128, 4, 2, 64, True, "fp32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_usp_matches_oracle(cp, case):
    layout, N, P, b, S, hq, hkv, d, causal, dt = case
    q, k, v = W.random_qkv(b, S, hq, hkv, d, dt, seed=S + 5 * N + P)
    o, lse = _usp(cp, q, k, v, layout, N, P, causal)
    ro, rl = oracle.usp_attention(np64(q), np64(k), np64(v), layout, N, P, causal, d ** -0.5)
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


@pytest.mark.parametrize("layout,N,P,b,S,hq,hkv,causal", [("zigzag", 2, 2, 1, 1024, 8, 4, True),
                                                          ("striped", 4, 2, 1, 1024, 8, 2, True),
                                                          ("contiguous", 3, 2, 2, 600, 4, 2, True),
                                                          ("zigzag", 2, 4, 1, 512, 8, 8, False)])
def test_usp_bwd_matches_oracle(cp, layout, N, P, b, S, hq, hkv, causal):
    d = 128
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "bf16", seed=S + 3 * N + P)
    do = W.random_do(b, S, hq, d, "bf16", seed=S + 3 * N + P)
    qr, kr, vr, dor = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v, do))
    o, lse = cp.usp_attn_fwd(qr, kr, vr, layout, N, P, causal)
    grads = cp.usp_attn_bwd(qr, kr, vr, o, lse, dor, layout, N, P, causal)
    grads = [cp.layout_permute(g, layout, N, inverse=True) for g in grads]
    cp.stream_check()
    want = oracle.usp_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, P, causal, d ** -0.5)
    for name, g, w in zip(("dq", "dk", "dv"), grads, want):
        err = np.max(np.abs(np64(g) - w))
        assert err <= 2e-2 * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))


@pytest.mark.parametrize("layout,N,P,d", [("zigzag", 2, 2, 64), ("contiguous", 1, 2, 128)])
def test_usp_bwd_fp32_matches_oracle(cp, layout, N, P, d):
    """fp32 through the FFMA backward (N = 1: plain Ulysses), 1e-4 x max |ref|."""
    b, S, hq, hkv = 1, 256, 4, 2
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "fp32", seed=S + N + d)
    do = W.random_do(b, S, hq, d, "fp32", seed=S + N + d)
    qr, kr, vr, dor = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v, do))
    o, lse = cp.usp_attn_fwd(qr, kr, vr, layout, N, P, True)
    grads = cp.usp_attn_bwd(qr, kr, vr, o, lse, dor, layout, N, P, True)
    grads = [cp.layout_permute(g, layout, N, inverse=True) for g in grads]
    cp.stream_check()
    want = oracle.usp_attention_bwd(np64(q), np64(k), np64(v), np64(do), layout, N, P, True, d ** -0.5)
    for name, g, w in zip(("dq", "dk", "dv"), grads, want):
        err = np.max(np.abs(np64(g) - w))
        assert err <= 1e-4 * np.max(np.abs(w)), (name, err, np.max(np.abs(w)))


def test_usp_argument_errors(cp):
    q, k, v = (t.cuda() for t in W.random_qkv(1, 256, 8, 2, 128, "bf16", seed=2))
    with pytest.raises(cp.CPError) as e:
        cp.usp_attn_fwd(q, k, v, "zigzag", 2, 4, True)    # 4 does not divide 2 kv heads
    assert e.value.code == 3
    with pytest.raises(cp.CPError) as e:
        cp.usp_attn_fwd(q, k, v, "zigzag", 3, 2, True)    # 256 % (3 * 2)
    assert e.value.code == 3
    o, lse = cp.usp_attn_fwd(q, k, v, "zigzag", 2, 2, True)
    with pytest.raises(cp.CPError) as e:
        cp.usp_attn_bwd(q, k, v, o.float(), lse, q, "zigzag", 2, 2, True)   # o in another dtype
    assert e.value.code == 3
    cp.stream_check()


def test_full_size_usp_sampled(cp):
    """The 8B workload's ring (zig-zag, N = 4) with Ulysses groups of P = 2 (8
    virtual ranks), at full size, the launch the bench times."""
    w = W.BY_NAME["llama3_8b_s8k_zigzag4"]
    q, k, v = W.make_inputs(w)
    o, lse = _usp(cp, q, k, v, w.layout, w.N, 2, w.causal)
    sel = sample_rows(w, n_random=24, seed=w.seed)
    q_sel = np.stack([np64(q[b, p, h]) for b, h, p in sel])
    ro, rl = oracle.attention_rows(q_sel, sel, np64(k), np64(v), w.causal, w.scale, w.hq)
    got_o = np.stack([np64(o[b, p, h]) for b, h, p in sel])
    got_l = np.array([float(lse[b, h, p]) for b, h, p in sel])
    tol_o, tol_l = TOL["bf16"]
    assert_close_lse(got_l, rl, tol_l)
    assert_close_o(got_o, ro, tol_o)
