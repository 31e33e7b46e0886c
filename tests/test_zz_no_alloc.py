"""The allocation-free ring entry point (cp_ring_attn_fwd_static_scratch).

Some callers cannot call cudaMalloc: a plug-in whose host engine owns all device
memory and hands it only input and output pointers, or a caller that must not take
the synchronisation an allocation can bring.  For them the library keeps the
stepwise ring's workspace in a static device array.  These tests check, through
the C ABI, that two calls in a row -- a larger problem, then a smaller one whose
workspace regions start at other offsets, so leftovers of the first call would be
read if the ring did not write every byte it reads -- give the same results as the
workspace-taking entry point within the parity tolerances, and agree with the fp64
oracle on sampled rows; and that problems too big for the static scratch are
refused before anything is launched.  This file is collected last so that a run
stopping at its first failure has run every other test.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = TOL["bf16"]
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _scratch_limit():
    """CP_STATIC_SCRATCH_BYTES as the public header defines it."""
    with open(os.path.join(ROOT, "include", "cpattn.h")) as f:
        m = re.search(r"#define CP_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", f.read())
    return int(m.group(1)) << int(m.group(2))


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _check_against_oracle(q, k, v, o_r, l_r, layout, N, n_rows, seed):
    """Sampled rows of the rank-major results against the fp64 oracle, row by row."""
    from oracle import layout as L
    b, S, hq, _ = q.shape
    rng = np.random.default_rng(seed)
    ranked = np.concatenate([np.array(L.rank_positions(layout, N, S, i)) for i in range(N)])
    rows = sorted({0, S - 1, *[int(x) for x in rng.integers(0, S, n_rows)]})
    sel = np.array([(0, int(rng.integers(hq)), int(ranked[r])) for r in rows], dtype=np.int64)
    q_sel = np.stack([np64(q[0, int(ranked[r]), h]) for r, (_, h, _) in zip(rows, sel)])
    ro, rl = oracle.attention_rows(q_sel, sel, np64(k), np64(v), True, 128 ** -0.5, hq)
    got_o = np.stack([np64(o_r[0, r, h]) for r, (_, h, _) in zip(rows, sel)])
    got_l = np.array([float(l_r[0, h, r]) for r, (_, h, _) in zip(rows, sel)])
    assert_close_lse(got_l, rl, TOL_LSE, "static scratch vs oracle")
    assert_close_o(got_o, ro, TOL_O, "static scratch vs oracle")


def test_static_scratch_matches_workspace_entry_twice(cp):
    limit = _scratch_limit()
    # larger first (K x 4: large leftovers), then smaller with other region offsets
    problems = [("zigzag", 4, 8192, 8, 2, 31, 4.0), ("striped", 8, 2048, 4, 4, 32, 1.0)]
    for layout, N, S, hq, hkv, seed, ks in problems:
        need = cp.ring_workspace_bytes(layout, N, "stepwise", 0, 1, S, hq, 128)
        assert 0 < need <= limit
        q, k, v = W.random_qkv(1, S, hq, hkv, 128, "bf16", seed=seed, k_scale=ks)
        qd, kd, vd = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v))
        ref_o, ref_l = cp.ring_attn_fwd(qd, kd, vd, layout, N, True, mode="stepwise")
        o = torch.empty_like(qd)
        lse = torch.empty((1, hq, S), dtype=torch.float32, device="cuda")
        cp.ring_attn_fwd_static_scratch(qd, kd, vd, layout, N, True, 128 ** -0.5, o, lse)
        cp.stream_check()
        assert torch.isfinite(lse).all()
        assert (o.float() - ref_o.float()).abs().max().item() <= TOL_O
        assert (lse - ref_l).abs().max().item() <= TOL_LSE
        _check_against_oracle(q, k, v, o, lse, layout, N, 24, seed)


def test_static_scratch_refuses_oversized_problems(cp):
    from context_attention_cp_b200._binding import CpTensor
    S, hq, d = 65536, 16, 128
    need = cp.ring_workspace_bytes("contiguous", 32, "stepwise", 0, 1, S, hq, d)
    assert need > _scratch_limit()

    def fake(shape, dtype):
        # no device memory behind it: the size check must refuse the call first, and
        # a NULL pointer is refused by the argument checks if it ever does not
        t = CpTensor()
        t.data, t.dtype = None, dtype
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
