"""GPU parity of Ulysses (cp_ulysses_all_to_all, cp_ulysses_attn_fwd) against the
oracle: the exchange bit for bit, the attention within the ring's tolerances (bf16
2e-2 on O and 1e-3 on lse; fp32 1e-4 and 1e-5)."""
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


@pytest.mark.parametrize("P,b,S,H,d,dt", [(4, 2, 64, 8, 128, "bf16"), (2, 1, 48, 6, 64, "fp32"), (8, 1, 8192, 32, 128, "bf16"),
                                        (1, 1, 16, 4, 128, "bf16"),
                                        # chunks of 2 16-byte pieces (one piece per thread) and of
                                        # 37 4-byte pieces (one warp per chunk, ragged last pass)
                                        (4, 1, 64, 4, 8, "fp32"), (2, 1, 32, 2, 37, "fp32"),
                                        # chunks of 20800 bytes: 8 KB segments, ragged last one
                                        (2, 1, 16, 4, 2600, "fp32")])
def test_all_to_all_is_bit_exact(cp, P, b, S, H, d, dt):
    x = torch.randn((b, S, H, d), generator=torch.Generator().manual_seed(S + P)).to(W.torch_dtype(dt))
    y = cp.ulysses_all_to_all(x.cuda(), P)
    bits = torch.int16 if dt == "bf16" else torch.int32
    want = oracle.ulysses_all_to_all(x.view(bits).numpy(), P)
    assert np.array_equal(y.cpu().view(bits).numpy().reshape(want.shape), want)
    back = cp.ulysses_all_to_all(y, P, inverse=True)
    assert torch.equal(back.cpu().view(bits), x.view(bits))


CASES = [
    # P, b, S, hq, hkv, d, causal, dtype
    (4, 1, 1024, 8, 4, 128, True, "bf16"),
    (2, 2, 600, 4, 2, 128, True, "bf16"),     # ragged query tiles per head group
    (8, 1, 512, 8, 8, 64, False, "bf16"),
    (1, 1, 256, 4, 1, 128, True, "bf16"),
    (2, 1, 128, 4, 2, 64, True, "fp32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_ulysses_matches_oracle(cp, case):
    P, b, S, hq, hkv, d, causal, dt = case
    q, k, v = W.random_qkv(b, S, hq, hkv, d, dt, seed=S + P)
    o, lse = cp.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P, causal)
    cp.stream_check()
    ro, rl = oracle.ulysses_attention(np64(q), np64(k), np64(v), P, causal, d ** -0.5)
    tol_o, tol_l = TOL[dt]
    assert_close_lse(np64(lse), rl, tol_l)
    assert_close_o(np64(o), ro, tol_o)


def test_ulysses_argument_errors(cp):
    q, k, v = (t.cuda() for t in W.random_qkv(1, 256, 8, 2, 128, "bf16", seed=2))
    with pytest.raises(cp.CPError) as e:
        cp.ulysses_attn_fwd(q, k, v, 4, True)      # 4 does not divide 2 kv heads
    assert e.value.code == 3
    with pytest.raises(cp.CPError) as e:
        cp.ulysses_attn_fwd(q, k, v, 3, True)
    assert e.value.code == 3


def test_full_size_ulysses_sampled(cp):
    """The 8B shape (32 query / 8 KV heads, S = 8192) with P = 4 at full size."""
    w = W.BY_NAME["llama3_8b_s8k_zigzag4"]
    q, k, v = W.make_inputs(w)
    o, lse = cp.ulysses_attn_fwd(q.cuda(), k.cuda(), v.cuda(), 4, True)
    cp.stream_check()
    sel = sample_rows(w, n_random=24, seed=w.seed)
    q_sel = np.stack([np64(q[b, p, h]) for b, h, p in sel])
    ro, rl = oracle.attention_rows(q_sel, sel, np64(k), np64(v), True, w.scale, w.hq)
    got_o = np.stack([np64(o[b, p, h]) for b, h, p in sel])
    got_l = np.array([float(lse[b, h, p]) for b, h, p in sel])
    tol_o, tol_l = TOL["bf16"]
    assert_close_lse(got_l, rl, tol_l)
    assert_close_o(got_o, ro, tol_o)


@pytest.mark.parametrize("P,b,S,hq,hkv,causal", [(4, 1, 1024, 8, 4, True), (2, 2, 600, 4, 2, True),
                                                 (8, 1, 512, 8, 8, False), (1, 1, 256, 4, 1, True)])
def test_ulysses_bwd_matches_oracle(cp, P, b, S, hq, hkv, causal):
    d = 128
    q, k, v = W.random_qkv(b, S, hq, hkv, d, "bf16", seed=S + 2 * P)
    do = W.random_do(b, S, hq, d, "bf16", seed=S + 2 * P)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = cp.ulysses_attn_fwd(qd, kd, vd, P, causal)
    dq, dk, dv = cp.ulysses_attn_bwd(qd, kd, vd, o, lse, dod, P, causal)
    cp.stream_check()
    want = oracle.ulysses_attention_bwd(np64(q), np64(k), np64(v), np64(do), P, causal, d ** -0.5)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        err = np.max(np.abs(np64(g) - w))
        assert err <= 2e-2 * np.max(np.abs(w)), (name, err)
