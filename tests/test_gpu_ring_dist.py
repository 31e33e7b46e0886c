"""The real-rank ring driver on the GPU.  Every GPU call of this project has one
device, and NCCL does not put two ranks on one device, so this runs a one-rank
NCCL group: the driver's default steps (the block kernel with its fused merge
epilogue; the block backward adding into fp32 accumulators) on cuda:0.  The
multi-rank exchange is covered on CPU (test_ring_dist)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", ["zigzag", "contiguous", "striped"])
def test_ring_dist_one_rank_on_gpu(layout):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from context_attention_cp_b200 import ring_dist
    port = 29400 + (os.getpid() + len(layout)) % 500
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1)
    try:
        torch.cuda.set_device(0)
        q, k, v = W.random_qkv(1, 512, 4, 2, 128, "bf16", seed=11)
        o, lse = ring_dist.ring_attn_fwd_dist(q.cuda(), k.cuda(), v.cuda(), layout, True)
        torch.cuda.synchronize()
        ro, rl = oracle.ring_attention(np64(q), np64(k), np64(v), layout, 1, True, 128 ** -0.5)
        tol_o, tol_l = TOL["bf16"]
        assert_close_lse(np64(lse), rl, tol_l)
        assert_close_o(np64(o), ro, tol_o)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dt,d", [("bf16", 128), ("fp32", 64)])
def test_ring_dist_bwd_one_rank_on_gpu(dt, d):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from context_attention_cp_b200 import ring_dist
    port = 29400 + (os.getpid() + d + 250) % 500
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1)
    try:
        torch.cuda.set_device(0)
        q, k, v = W.random_qkv(1, 384, 4, 2, d, dt, seed=13)
        do = W.random_do(1, 384, 4, d, dt, seed=13)
        qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
        o, lse = ring_dist.ring_attn_fwd_dist(qd, kd, vd, "zigzag", True)
        dq, dk, dv = ring_dist.ring_attn_bwd_dist(qd, kd, vd, o, lse, dod, "zigzag", True)
        torch.cuda.synchronize()
        want = oracle.attention_bwd(np64(q), np64(k), np64(v), np64(do), True, d ** -0.5)[:3]
        tol = 1e-4 if dt == "fp32" else 2e-2
        for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
            assert g.dtype == q.dtype
            err = np.max(np.abs(np64(g) - w))
            assert err <= tol * np.max(np.abs(w)), (name, err)
    finally:
        dist.destroy_process_group()
