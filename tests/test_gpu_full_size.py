"""Parity at the named workloads' full sizes, in the launch configuration the
benchmark times (fused ring, rank-major inputs): sampled output rows against the
fp64 oracle computed row by row (rows are independent, so each sampled row is
exact), plus whole-tensor properties (finite outputs, lse >= max over sampled)."""
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


def _run(cp, w, mode):
    q, k, v = W.make_inputs(w)
    qd, kd, vd = (cp.layout_permute(t.cuda(), w.layout, w.N) for t in (q, k, v))
    o, lse = cp.ring_attn_fwd(qd, kd, vd, w.layout, w.N, w.causal, w.scale, mode=mode)
    o = cp.layout_permute(o, w.layout, w.N, inverse=True)
    lse = cp.layout_permute(lse, w.layout, w.N, seq_axis=2, inverse=True)
    cp.stream_check()
    return q, k, v, o, lse


@pytest.mark.parametrize("name,mode", [
    ("llama3_8b_s8k_zigzag4", "fused"),
    ("llama3_8b_s8k_zigzag4", "stepwise"),
    ("s32k_b2_striped8_kx4", "fused"),
    ("llama3_70b_s128k_zigzag8", "fused"),
    ("noncausal_s64k_contig32", "fused"),
    ("noncausal_s64k_contig32", "stepwise"),
])
def test_full_size_sampled_rows(cp, name, mode):
    w = W.BY_NAME[name]
    q, k, v, o, lse = _run(cp, w, mode)
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()
    sel = sample_rows(w, n_random=24, seed=w.seed)
    q_sel = np.stack([np64(q[b, p, h]) for b, h, p in sel])
    ro, rl = oracle.attention_rows(q_sel, sel, np64(k), np64(v), w.causal, w.scale, w.hq)
    got_o = np.stack([np64(o[b, p, h]) for b, h, p in sel])
    got_l = np.array([float(lse[b, h, p]) for b, h, p in sel])
    tol_o, tol_l = TOL[w.dtype]
    assert_close_lse(got_l, rl, tol_l, name)
    assert_close_o(got_o, ro, tol_o, name)
    del q, k, v, o, lse
    torch.cuda.empty_cache()
