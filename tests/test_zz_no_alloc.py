"""The allocation-free ring entry point (cp_ring_attn_fwd_static_scratch).

Some callers cannot call cudaMalloc: a plug-in whose host engine owns all device
memory and hands it only input and output pointers, or a caller that must not take
the synchronisation an allocation can bring.  For them the library keeps the
stepwise ring's workspace in a static device array.  These tests check, through
the C ABI, that two calls in a row give the same results as the workspace-taking
entry point (within the parity tolerances), and that problems too big for the
static scratch are refused before anything is launched.  This file is collected
last so that a run stopping at its first failure has run every other test.
"""
import ctypes

import pytest
import torch

import cp_workloads as W

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _problem(cp, layout, N, S, hq, hkv, seed):
    q, k, v = W.random_qkv(1, S, hq, hkv, 128, "bf16", seed=seed)
    return [cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v)]


def test_static_scratch_matches_workspace_entry_twice(cp):
    problems = [("zigzag", 4, 2048, 8, 2, 31), ("striped", 8, 4096, 4, 4, 32)]
    for layout, N, S, hq, hkv, seed in problems:
        q, k, v = _problem(cp, layout, N, S, hq, hkv, seed)
        ref_o, ref_l = cp.ring_attn_fwd(q, k, v, layout, N, True, mode="stepwise")
        o = torch.empty_like(q)
        lse = torch.empty((1, hq, S), dtype=torch.float32, device="cuda")
        cp.ring_attn_fwd_static_scratch(q, k, v, layout, N, True, 128 ** -0.5, o, lse)
        cp.stream_check()
        assert (o.float() - ref_o.float()).abs().max().item() <= TOL_O
        assert (lse - ref_l).abs().max().item() <= TOL_LSE
        assert torch.isfinite(lse).all()


def test_static_scratch_refuses_oversized_problems(cp):
    from context_attention_cp_b200._binding import CpTensor
    S, hq, d = 65536, 16, 128
    need = cp.ring_workspace_bytes("contiguous", 32, "stepwise", 0, 1, S, hq, d)
    assert need > (64 << 20)

    def fake(shape, dtype):
        t = CpTensor()
        t.data, t.dtype = 0x10000, dtype
        acc = 1
        for i in (3, 2, 1, 0):
            t.shape[i], t.stride[i] = shape[i], acc
            acc *= shape[i]
        return t

    q = fake([1, S, hq, d], 0)
    o = fake([1, S, hq, d], 0)
    lse = fake([1, hq, S, 1], 1)
    rc = cp.lib().cp_ring_attn_fwd_static_scratch(0, 32, 0, ctypes.byref(q), ctypes.byref(q), ctypes.byref(q),
                                                  ctypes.c_float(0.088), ctypes.byref(o), ctypes.byref(lse), None)
    assert rc == 2
    assert b"static scratch" in cp.lib().cp_last_error()
