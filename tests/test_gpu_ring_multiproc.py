"""The real-rank ring driver (context_attention_cp_b200.ring_dist) with several
ranks and the real CUDA kernels: 2 and 4 processes, each with its own CUDA context
on cuda:0, form a gloo group ("上下文并行与 Ring Attention", section Ring Attention:
each rank holds its Q and attends it to the K/V block it holds, passing the block
on to the next rank while the block kernel runs; section 分块注意力 for the
backward, dK / dV travelling with their block).

The K/V blocks and the travelling dK / dV accumulators are held in host memory and
exchanged by gloo (this stands in for the NCCL transfers between GPUs: every call
of this project has one GPU); every compute step copies the held block to the GPU
and runs the library's block kernels there (cp_block_attn_fwd with its fused merge,
the standalone merge for the last step, cp_block_attn_bwd on the tensor cores).
No kernel waits on another process: the ranks synchronise only on the host.  The
results are compared with the fp64 oracle's whole-sequence attention and gradients.
"""
import os
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, layout, S, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    import cp_workloads as W
    import oracle
    from context_attention_cp_b200 import _binding as B
    from context_attention_cp_b200 import ring_dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        hq, hkv, d = 4, 1, 128
        q, k, v = W.random_qkv(1, S, hq, hkv, d, "bf16", seed=S + world)
        do = W.random_do(1, S, hq, d, "bf16", seed=S + world)
        pos = torch.tensor(oracle.layout.rank_positions(layout, world, S, rank))
        ql, kl, vl, dol = (t[:, pos].contiguous() for t in (q, k, v, do))

        def fwd_step(qq, kk, vv, q_range, kv_range, causal, scale, o, lse, accumulate):
            ring_dist.block_compute(qq, kk.cuda(), vv.cuda(), q_range, kv_range, causal, scale, o, lse, accumulate)

        def bwd_step(qq, kk, vv, oo, ll, gg, q_range, kv_range, causal, scale, dq, dk, dv):
            dk_g, dv_g = dk.cuda(), dv.cuda()
            B.block_attn_bwd(qq, kk.cuda(), vv.cuda(), oo, ll, gg, q_range, kv_range, causal, scale, dq, dk_g, dv_g)
            dk.copy_(dk_g.cpu())
            dv.copy_(dv_g.cpu())

        qg, dog = ql.cuda(), dol.cuda()
        o, lse = ring_dist.ring_attn_fwd_dist(qg, kl, vl, layout, True, compute=fwd_step)
        dq, dk, dv = ring_dist.ring_attn_bwd_dist(qg, kl, vl, o, lse, dog, layout, True, compute=bwd_step)
        torch.cuda.synchronize()
        B.stream_check()
        p = pos.numpy()
        want_o, want_l = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), True,
                                          d ** -0.5)
        wg = oracle.attention_bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                                  True, d ** -0.5)[:3]
        f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
        errs = {"o": float(np.max(np.abs(f(o) - want_o[:, p]))),
                "lse": float(np.max(np.abs(f(lse) - want_l[:, :, p])))}
        for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), wg):
            errs[name] = float(np.max(np.abs(f(g) - w[:, p])) / np.max(np.abs(w)))
        out[rank] = errs
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S", [("zigzag", 2, 1024), ("striped", 4, 1024), ("zigzag", 4, 2048)])
def test_ring_dist_processes_share_one_gpu(layout, world, S):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.multiprocessing as mp
    port = 29700 + (os.getpid() + world * 11 + S) % 800
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, layout, S, out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    errs = dict(out)
    for rank, e in errs.items():
        assert e["o"] <= 2e-2 and e["lse"] <= 1e-3, errs          # the bf16 forward bar
        assert max(e["dq"], e["dk"], e["dv"]) <= 2e-2, errs       # the tensor-core backward bar


def _peer_worker(rank, world, port, layout, S, causal, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    import cp_workloads as W
    import oracle
    from context_attention_cp_b200 import _binding as B
    from context_attention_cp_b200 import ring_dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        hq, hkv, d = 4, 1, 128
        q, k, v = W.random_qkv(1, S, hq, hkv, d, "bf16", seed=S + world + 1)
        do = W.random_do(1, S, hq, d, "bf16", seed=S + world + 1)
        pos = torch.tensor(oracle.layout.rank_positions(layout, world, S, rank))
        ql, kl, vl, dol = (t[:, pos].contiguous() for t in (q, k, v, do))
        kv = ring_dist.PeerBlocks([kl.shape, vl.shape], torch.bfloat16, "cuda")
        acc = ring_dist.PeerBlocks([kl.shape, vl.shape], torch.float32, "cuda")
        # every other rank's block is a mapping of that process's memory, not a copy
        mapped = all(kv.views[t][j].data_ptr() != kv.local[t].data_ptr()
                     for t in range(2) for j in range(world) if j != rank)
        p = pos.numpy()
        errs, gerrs = [], []
        f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
        # the blocks rewritten between two calls (x2 is exact in bf16); each forward runs
        # twice, pulling the peer blocks into local buffers one step ahead and reading
        # them in place: the same kernels on the same bytes, so the results must agree
        # bit for bit
        same = True
        for k_scale in (1.0, 2.0):
            kv.local[0].copy_((kl * k_scale).cuda())
            kv.local[1].copy_(vl.cuda())
            o, lse = ring_dist.ring_attn_fwd_peer(ql.cuda(), kv, layout, causal, stage=True)
            o2, lse2 = ring_dist.ring_attn_fwd_peer(ql.cuda(), kv, layout, causal, stage=False)
            B.stream_check()
            same = same and torch.equal(o, o2) and torch.equal(lse, lse2)
            k64 = k.double().numpy() * k_scale
            want_o, want_l = oracle.attention(q.double().numpy(), k64, v.double().numpy(), causal, d ** -0.5)
            errs.append((float(np.max(np.abs(f(o) - want_o[:, p]))), float(np.max(np.abs(f(lse) - want_l[:, :, p])))))
            # the backward adds into the owners' dK, dV accumulators where they lie
            dq, dk, dv = ring_dist.ring_attn_bwd_peer(ql.cuda(), kv, o, lse, dol.cuda(), layout, causal, acc=acc)
            B.stream_check()
            wg = oracle.attention_bwd(q.double().numpy(), k64, v.double().numpy(), do.double().numpy(), causal,
                                      d ** -0.5)[:3]
            gerrs.append([float(np.max(np.abs(f(g) - w[:, p])) / np.max(np.abs(w))) for g, w in zip((dq, dk, dv), wg)])
        acc.close()
        kv.close()
        out[rank] = (errs, gerrs, mapped, same)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S,causal", [("zigzag", 2, 1024, True), ("striped", 4, 1024, True),
                                                   ("zigzag", 4, 2048, True), ("contiguous", 3, 1536, True),
                                                   ("contiguous", 2, 1024, False)])
def test_peer_ring_processes_share_one_gpu(layout, world, S, causal):
    """The ring without sends (ring_dist.ring_attn_fwd_peer, ring_attn_bwd_peer): each
    process maps the other processes' K/V blocks and dK/dV accumulators
    (cp_peer_export / cp_peer_import, CUDA IPC); the forward pulls each peer block
    into a local double buffer one step ahead (cp_peer_copy on a copy stream) or
    reads it in place -- bit for bit the same result -- and the backward's kernels
    read the K/V and add into the accumulators where they lie; no rank sends
    anything.  The processes
    share cuda:0, so the mapped memory is the same GPU's: this checks the mapping,
    the schedule and the kernels, not NVLink.  No kernel waits on another process:
    the ranks meet only on the host (publish / release)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.multiprocessing as mp
    port = 29300 + (os.getpid() + world * 13 + S + int(causal)) % 250
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_peer_worker, args=(world, port, layout, S, causal, out), nprocs=world, start_method="spawn",
                       join=True)
    assert sorted(out.keys()) == list(range(world))
    res = dict(out)
    for rank, (errs, gerrs, mapped, same) in res.items():
        assert mapped and same, res
        for err_o, err_l in errs:
            assert err_o <= 2e-2 and err_l <= 1e-3, res   # the bf16 forward bar
        for g in gerrs:
            assert max(g) <= 2e-2, res                    # the tensor-core backward bar
