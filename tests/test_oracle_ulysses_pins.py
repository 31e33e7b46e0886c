"""Pins for the oracle's Ulysses form (section DeepSpeed-Ulysses): the exchange is a
bijection that puts block (s_i, h_j) on rank j, its inverse undoes it, and the
page's four steps around per-head-group attention give plain attention."""
import numpy as np
import pytest

import oracle


def test_all_to_all_places_blocks_and_inverts():
    b, S, H, d, P = 2, 12, 8, 3, 4
    x = np.arange(b * S * H * d, dtype=np.float64).reshape(b, S, H, d)
    y = oracle.ulysses_all_to_all(x, P)
    c, hp = S // P, H // P
    for i in range(P):
        for j in range(P):
            assert np.array_equal(y[j, :, i * c:(i + 1) * c], x[:, i * c:(i + 1) * c, j * hp:(j + 1) * hp])
    assert np.array_equal(oracle.ulysses_all_to_all(y, P, inverse=True), x)
    assert sorted(y.ravel().tolist()) == sorted(x.ravel().tolist())


@pytest.mark.parametrize("P,causal", [(1, True), (2, True), (4, False), (4, True)])
def test_steps_equal_plain_attention(P, causal):
    r = np.random.default_rng(P + causal)
    b, S, hq, hkv, d = 2, 16, 8, 4, 5
    q, k, v = r.standard_normal((b, S, hq, d)), r.standard_normal((b, S, hkv, d)), r.standard_normal((b, S, hkv, d))
    o, lse = oracle.ulysses_attention_steps(q, k, v, P, causal, 0.45)
    ow, lw = oracle.ulysses_attention(q, k, v, P, causal, 0.45)
    assert np.max(np.abs(o - ow)) <= 1e-13
    assert np.max(np.abs(lse - lw)) <= 1e-13


def test_p_must_divide_heads():
    x = np.zeros((1, 8, 6, 2))
    with pytest.raises(ValueError):
        oracle.ulysses_attention(x, x[:, :, :3], x[:, :, :3], 4, True, 0.5)


@pytest.mark.parametrize("P", [1, 2, 4])
def test_backward_steps_equal_plain_gradients(P):
    r = np.random.default_rng(10 + P)
    b, S, hq, hkv, d = 1, 12, 8, 4, 3
    q, k, v, do = (r.standard_normal(s) for s in ((b, S, hq, d), (b, S, hkv, d), (b, S, hkv, d), (b, S, hq, d)))
    got = oracle.ulysses_attention_bwd_steps(q, k, v, do, P, True, 0.6)
    want = oracle.ulysses_attention_bwd(q, k, v, do, P, True, 0.6)
    for g, w in zip(got, want):
        assert np.max(np.abs(g - w)) <= 1e-13
