"""Parity at the named workloads' full sizes, in the launch configuration the
benchmark times (rank-major inputs; the fused ring, and the stepwise forms of the
ring): sampled output rows against the fp64 oracle computed row by row (rows are
independent, so each sampled row is exact) -- position 0, every chunk and rank
boundary, and at least one row of every (batch, query head) -- plus properties
that hold at any size: finite outputs, and with Q = 0 the number of keys every
row sees, read back from lse and compared bit-exactly with its closed form."""
import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64, sample_rows

pytestmark = pytest.mark.gpu

_INPUTS = {}


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    yield m
    _INPUTS.clear()


def _inputs(w):
    """The workload's CPU inputs, drawn once per module (the largest takes seconds)."""
    if w.name not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[w.name] = W.make_inputs(w)
    return _INPUTS[w.name]


def _run(cp, w, mode, q, k, v):
    qd, kd, vd = (cp.layout_permute(t.cuda(), w.layout, w.N) for t in (q, k, v))
    o, lse = cp.ring_attn_fwd(qd, kd, vd, w.layout, w.N, w.causal, w.scale, mode=mode)
    del qd, kd, vd
    o = cp.layout_permute(o, w.layout, w.N, inverse=True)
    lse = cp.layout_permute(lse, w.layout, w.N, seq_axis=2, inverse=True)
    cp.stream_check()
    return o, lse


def _rows_every_head(w, seed):
    """sample_rows' boundary and random rows, plus one random position for every
    (batch, query head)."""
    rng = np.random.default_rng(seed + 1)
    extra = [(b, h, int(rng.integers(w.S))) for b in range(w.b) for h in range(w.hq)]
    return np.concatenate([sample_rows(w, n_random=24, seed=w.seed), np.array(extra, dtype=np.int64)])


@pytest.mark.parametrize("name,mode", [
    ("llama3_8b_s8k_zigzag4", "fused"),
    ("llama3_8b_s8k_zigzag4", "stepwise"),
    ("llama3_8b_s8k_zigzag4", "stepwise_epi"),
    ("s32k_b2_striped8_kx4", "fused"),
    ("s32k_b2_striped8_kx4", "stepwise"),
    ("s32k_b2_striped8_kx4", "stepwise_epi"),
    ("llama3_70b_s128k_zigzag8", "fused"),
    ("llama3_70b_s128k_zigzag8", "stepwise"),
    ("llama3_70b_s128k_zigzag8", "stepwise_epi"),
    ("noncausal_s64k_contig32", "fused"),
    ("noncausal_s64k_contig32", "stepwise"),
    ("noncausal_s64k_contig32", "stepwise_epi"),
])
def test_full_size_sampled_rows(cp, name, mode):
    w = W.BY_NAME[name]
    q, k, v = _inputs(w)
    o, lse = _run(cp, w, mode, q, k, v)
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()
    sel = _rows_every_head(w, w.seed)
    q_sel = np.stack([np64(q[b, p, h]) for b, h, p in sel])
    ro, rl = oracle.attention_rows(q_sel, sel, np64(k), np64(v), w.causal, w.scale, w.hq)
    got_o = np.stack([np64(o[b, p, h]) for b, h, p in sel])
    got_l = np.array([float(lse[b, h, p]) for b, h, p in sel])
    tol_o, tol_l = TOL[w.dtype]
    assert_close_lse(got_l, rl, tol_l, name)
    assert_close_o(got_o, ro, tol_o, name)
    del o, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["llama3_8b_s8k_zigzag4", "s32k_b2_striped8_kx4", "llama3_70b_s128k_zigzag8",
                                  "noncausal_s64k_contig32"])
def test_full_size_mask_counts_with_zero_queries(cp, name):
    """Q = 0: every score is 0, every probability exactly 1, so e^{lse} is the number
    of keys the row sees: p + 1 for the causal mask at original position p, S
    without it.  Checked for every (batch, head, row) of the full-size fused ring,
    which pins the mask, the tile skipping and the merge of the ring steps
    bit-exactly at the benchmarked size."""
    w = W.BY_NAME[name]
    _, k, v = _inputs(w)
    kd, vd = (cp.layout_permute(t.cuda(), w.layout, w.N) for t in (k, v))
    qd = torch.zeros((w.b, w.S, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    o, lse = cp.ring_attn_fwd(qd, kd, vd, w.layout, w.N, w.causal, w.scale)
    del qd, kd, vd, o
    lse = cp.layout_permute(lse, w.layout, w.N, seq_axis=2, inverse=True)
    cp.stream_check()
    counts = torch.exp(lse.double()).round().long()
    want = (torch.arange(1, w.S + 1, device="cuda") if w.causal else torch.full((w.S,), w.S, device="cuda"))
    bad = (counts != want.view(1, 1, -1)).sum().item()
    assert bad == 0, "%d rows with a wrong count of visible keys" % bad
    del lse, counts
    torch.cuda.empty_cache()
