"""The real-rank ring (context_attention_cp_b200.ring_dist) on CPU: 2, 3 and 4 gloo
ranks, each holding only its own layout block, pass K/V around the ring
(section Ring Attention).  The block step is injected: here the fp64 oracle's block
attention and LSE merge, so the test checks the schedule (which block each rank
holds at each step, the exchange, the buffer swap) and the step-by-step merge
against the oracle's whole-sequence attention."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _positions(rng_tuple):
    starts, lens, stride = rng_tuple
    out = []
    for s0, n in zip(starts, lens):
        out.extend(s0 + t * stride for t in range(n))
    return np.array(out, dtype=np.int64)


def _oracle_merge(o_acc, lse_acc, o_b, lse_b, o_out):
    """The last step's merge of the driver, done by the oracle: (o_acc, lse_acc) and
    (o_b, lse_b) merged, o written to o_out, lse_acc updated."""
    import oracle
    om, lm = oracle.lse_merge(o_acc.numpy().transpose(0, 2, 1, 3), lse_acc.numpy(),
                              o_b.numpy().transpose(0, 2, 1, 3), lse_b.numpy())
    o_out.copy_(torch.from_numpy(np.ascontiguousarray(om.transpose(0, 2, 1, 3))))
    lse_acc.copy_(torch.from_numpy(np.ascontiguousarray(lm)))


def _worker(rank, world, port, layout, S, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from context_attention_cp_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = np.random.default_rng(7)
        b, hq, hkv, d = 1, 4, 2, 8
        q = r.standard_normal((b, S, hq, d))
        k = r.standard_normal((b, S, hkv, d))
        v = r.standard_normal((b, S, hkv, d))
        pos = np.array(oracle.layout.rank_positions(layout, world, S, rank))
        ql, kl, vl = (torch.from_numpy(np.ascontiguousarray(t[:, pos])) for t in (q, k, v))
        seen = []

        def oracle_step(qq, kk, vv, q_range, kv_range, causal, scale, o, lse, accumulate):
            pk = _positions(kv_range)
            seen.append(int(pk[0]))
            ob, lb = oracle.attention(qq.numpy(), kk.numpy(), vv.numpy(), causal, scale,
                                      pos_q=_positions(q_range), pos_k=pk, nthreads=1)
            if accumulate:
                om, lm = oracle.lse_merge(o.numpy().transpose(0, 2, 1, 3), lse.numpy(), ob.transpose(0, 2, 1, 3), lb)
                ob, lb = om.transpose(0, 2, 1, 3), lm
            o.copy_(torch.from_numpy(np.ascontiguousarray(ob)))
            lse.copy_(torch.from_numpy(np.ascontiguousarray(lb)))

        k_before, v_before = kl.clone(), vl.clone()
        o, lse = ring_dist.ring_attn_fwd_dist(ql, kl, vl, layout, True, 0.35, compute=oracle_step,
                                              merge=_oracle_merge)
        # the caller's blocks are read, never written (they feed the backward next)
        assert torch.equal(kl, k_before) and torch.equal(vl, v_before)
        want_o, want_l = oracle.ring_attention(q, k, v, layout, world, True, 0.35, nthreads=1)
        out[rank] = (float(np.max(np.abs(o.numpy() - want_o[:, pos]))),
                     float(np.max(np.abs(lse.numpy() - want_l[:, :, pos]))),
                     seen,
                     [int(oracle.layout.rank_positions(layout, world, S, (rank - s) % world)[0]) for s in range(world)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S", [("zigzag", 2, 32), ("striped", 4, 32), ("contiguous", 3, 24),
                                            ("zigzag", 4, 64)])
def test_ring_over_gloo_ranks(layout, world, S):
    port = 29600 + (os.getpid() + world * 7 + len(layout)) % 900
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, layout, S, out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank, (err_o, err_l, seen, want_seen) in out.items():
        assert err_o <= 1e-6 and err_l <= 1e-6, (rank, err_o, err_l)
        assert seen == want_seen, (rank, seen, want_seen)   # step r holds rank (i - r) mod N's block


def _bwd_worker(rank, world, port, layout, S, causal, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from context_attention_cp_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = np.random.default_rng(11)
        b, hq, hkv, d = 1, 4, 2, 8
        q = r.standard_normal((b, S, hq, d))
        k = r.standard_normal((b, S, hkv, d))
        v = r.standard_normal((b, S, hkv, d))
        do = r.standard_normal((b, S, hq, d))
        o_full, lse_full = oracle.attention(q, k, v, causal, 0.35, nthreads=1)
        pos = np.array(oracle.layout.rank_positions(layout, world, S, rank))
        loc = lambda t: torch.from_numpy(np.ascontiguousarray(t[:, pos]))  # noqa: E731
        ql, kl, vl, dol, ol = (loc(t) for t in (q, k, v, do, o_full))
        lsel = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, pos]))
        seen = []

        def oracle_step(qq, kk, vv, oo, ll, gg, q_range, kv_range, causal, scale, dq, dk, dv):
            pk = _positions(kv_range)
            seen.append(int(pk[0]))
            delta = np.einsum("bshd,bshd->bhs", gg.numpy(), oo.numpy())
            a, bk, bv, _, _ = oracle.attention_bwd(qq.numpy(), kk.numpy(), vv.numpy(), gg.numpy(), causal, scale,
                                                   pos_q=_positions(q_range), pos_k=pk, lse=ll.numpy(), delta=delta,
                                                   nthreads=1)
            dq += torch.from_numpy(a)
            dk += torch.from_numpy(bk)
            dv += torch.from_numpy(bv)

        k_before, v_before = kl.clone(), vl.clone()
        dq, dk, dv = ring_dist.ring_attn_bwd_dist(ql, kl, vl, ol, lsel, dol, layout, causal, 0.35, compute=oracle_step)
        assert torch.equal(kl, k_before) and torch.equal(vl, v_before)
        want = oracle.attention_bwd(q, k, v, do, causal, 0.35, nthreads=1)[:3]
        errs = [float(np.max(np.abs(g.numpy() - w[:, pos]))) for g, w in zip((dq, dk, dv), want)]
        out[rank] = (errs, seen,
                     [int(oracle.layout.rank_positions(layout, world, S, (rank - s) % world)[0]) for s in range(world)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S,causal", [("zigzag", 2, 32, True), ("striped", 4, 32, True),
                                                   ("contiguous", 3, 24, True), ("zigzag", 1, 16, True),
                                                   ("contiguous", 2, 16, False)])
def test_ring_bwd_over_gloo_ranks(layout, world, S, causal):
    """Every rank ends with the whole-sequence gradients of its own rows and keys:
    dQ accumulated locally, dK and dV carried around the ring with their block and
    brought home after the last step."""
    port = 29600 + (os.getpid() + world * 13 + len(layout) + 450 + 7 * causal) % 900
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_bwd_worker, args=(world, port, layout, S, causal, out), nprocs=world, start_method="spawn",
                       join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank, (errs, seen, want_seen) in out.items():
        assert max(errs) <= 1e-6, (rank, errs)   # the driver's accumulators are fp32
        assert seen == want_seen, (rank, seen, want_seen)


def _group_worker(rank, world, port, out):
    """Ranks 1 and 3 of 4 form a sub-group and run the ring (forward and backward)
    inside it: the driver must address its neighbours by their global ranks."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from context_attention_cp_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sub = dist.new_group([1, 3])
        if rank in (1, 3):
            me, n = [1, 3].index(rank), 2
            S, layout = 16, "zigzag"
            r = np.random.default_rng(5)
            q, k, v, do = (r.standard_normal(s) for s in ((1, S, 2, 4), (1, S, 1, 4), (1, S, 1, 4), (1, S, 2, 4)))
            pos = np.array(oracle.layout.rank_positions(layout, n, S, me))
            loc = lambda t: torch.from_numpy(np.ascontiguousarray(t[:, pos]))  # noqa: E731

            def fwd_step(qq, kk, vv, q_range, kv_range, causal, scale, o, lse, accumulate):
                ob, lb = oracle.attention(qq.numpy(), kk.numpy(), vv.numpy(), causal, scale,
                                          pos_q=_positions(q_range), pos_k=_positions(kv_range), nthreads=1)
                if accumulate:
                    om, lm = oracle.lse_merge(o.numpy().transpose(0, 2, 1, 3), lse.numpy(), ob.transpose(0, 2, 1, 3), lb)
                    ob, lb = om.transpose(0, 2, 1, 3), lm
                o.copy_(torch.from_numpy(np.ascontiguousarray(ob)))
                lse.copy_(torch.from_numpy(np.ascontiguousarray(lb)))

            def bwd_step(qq, kk, vv, oo, ll, gg, q_range, kv_range, causal, scale, dq, dk, dv):
                delta = np.einsum("bshd,bshd->bhs", gg.numpy(), oo.numpy())
                a, bk, bv, _, _ = oracle.attention_bwd(qq.numpy(), kk.numpy(), vv.numpy(), gg.numpy(), causal, scale,
                                                       pos_q=_positions(q_range), pos_k=_positions(kv_range),
                                                       lse=ll.numpy(), delta=delta, nthreads=1)
                dq += torch.from_numpy(a)
                dk += torch.from_numpy(bk)
                dv += torch.from_numpy(bv)

            o, lse = ring_dist.ring_attn_fwd_dist(loc(q), loc(k), loc(v), layout, True, 0.5, group=sub,
                                                  compute=fwd_step, merge=_oracle_merge)
            grads = ring_dist.ring_attn_bwd_dist(loc(q), loc(k), loc(v), o, lse, loc(do), layout, True, 0.5,
                                                 group=sub, compute=bwd_step)
            wo, wl = oracle.attention(q, k, v, True, 0.5, nthreads=1)
            wg = oracle.attention_bwd(q, k, v, do, True, 0.5, nthreads=1)[:3]
            errs = [float(np.max(np.abs(o.numpy() - wo[:, pos]))), float(np.max(np.abs(lse.numpy() - wl[:, :, pos])))]
            errs += [float(np.max(np.abs(g.numpy() - w[:, pos]))) for g, w in zip(grads, wg)]
            out[rank] = errs
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ring_in_a_sub_group():
    port = 29600 + (os.getpid() + 777) % 900
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_group_worker, args=(4, port, out), nprocs=4, start_method="spawn", join=True)
    assert sorted(out.keys()) == [1, 3]
    for rank, errs in out.items():
        assert max(errs) <= 1e-6, (rank, errs)


def _peer_worker(rank, world, port, layout, S, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from context_attention_cp_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = np.random.default_rng(5)
        b, hq, hkv, d = 1, 4, 2, 8
        q = r.standard_normal((b, S, hq, d))
        k = r.standard_normal((b, S, hkv, d))
        v = r.standard_normal((b, S, hkv, d))
        pos = np.array(oracle.layout.rank_positions(layout, world, S, rank))
        ql, kl, vl = (torch.from_numpy(np.ascontiguousarray(t[:, pos])) for t in (q, k, v))
        seen = []

        def oracle_step(qq, kk, vv, q_range, kv_range, causal, scale, o, lse, accumulate):
            pk = _positions(kv_range)
            seen.append(int(pk[0]))
            ob, lb = oracle.attention(qq.numpy(), kk.numpy(), vv.numpy(), causal, scale,
                                      pos_q=_positions(q_range), pos_k=pk, nthreads=1)
            if accumulate:
                om, lm = oracle.lse_merge(o.numpy().transpose(0, 2, 1, 3), lse.numpy(), ob.transpose(0, 2, 1, 3), lb)
                ob, lb = om.transpose(0, 2, 1, 3), lm
            o.copy_(torch.from_numpy(np.ascontiguousarray(ob)))
            lse.copy_(torch.from_numpy(np.ascontiguousarray(lb)))

        kv = ring_dist.PeerBlocks([kl.shape, vl.shape], kl.dtype, "cpu")
        errs = []
        # two calls over the same blocks, rewritten between them: the first pulls each
        # peer block into a local buffer one step ahead, the second reads it in place
        for scale, stage in ((0.35, True), (0.2, False)):
            kv.local[0].copy_(kl * (scale / 0.35))
            kv.local[1].copy_(vl)
            seen.clear()
            o, lse = ring_dist.ring_attn_fwd_peer(ql, kv, layout, True, 0.35, stage=stage, compute=oracle_step,
                                                  merge=_oracle_merge)
            want_o, want_l = oracle.ring_attention(q, k * (scale / 0.35), v, layout, world, True, 0.35, nthreads=1)
            errs.append((float(np.max(np.abs(o.numpy() - want_o[:, pos]))),
                         float(np.max(np.abs(lse.numpy() - want_l[:, :, pos])))))
        kv.close()
        out[rank] = (errs, seen,
                     [int(oracle.layout.rank_positions(layout, world, S, (rank - s) % world)[0]) for s in range(world)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S", [("zigzag", 2, 32), ("striped", 3, 24), ("zigzag", 4, 64),
                                            ("contiguous", 5, 40)])
def test_peer_ring_over_gloo_ranks(layout, world, S):
    """The ring without sends (ring_attn_fwd_peer): no rank sends a block; step r
    attends to rank (i - r) mod N's K/V block, pulled into a local double buffer one
    step ahead or read where it lies (on CPU ranks the blocks live in shared memory
    that every rank opens, standing in for the device mapping), twice over blocks
    rewritten between the calls; 5 ranks cycle the two buffers twice."""
    port = 29550 + (os.getpid() + world * 5 + S) % 900
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_peer_worker, args=(world, port, layout, S, out), nprocs=world, start_method="spawn",
                       join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank, (errs, seen, want_seen) in out.items():
        for err_o, err_l in errs:
            assert err_o <= 1e-6 and err_l <= 1e-6, (rank, errs)
        assert seen == want_seen, (rank, seen, want_seen)


def _peer_bwd_worker(rank, world, port, layout, S, causal, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from context_attention_cp_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r = np.random.default_rng(13)
        b, hq, hkv, d = 1, 4, 2, 8
        q = r.standard_normal((b, S, hq, d))
        k = r.standard_normal((b, S, hkv, d))
        v = r.standard_normal((b, S, hkv, d))
        do = r.standard_normal((b, S, hq, d))
        o_full, lse_full = oracle.attention(q, k, v, causal, 0.35, nthreads=1)
        pos = np.array(oracle.layout.rank_positions(layout, world, S, rank))
        loc = lambda t: torch.from_numpy(np.ascontiguousarray(t[:, pos]))  # noqa: E731
        ql, kl, vl, dol, ol = (loc(t) for t in (q, k, v, do, o_full))
        lsel = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, pos]))
        seen = []

        def oracle_step(qq, kk, vv, oo, ll, gg, q_range, kv_range, causal, scale, dq, dk, dv):
            pk = _positions(kv_range)
            seen.append(int(pk[0]))
            delta = np.einsum("bshd,bshd->bhs", gg.numpy(), oo.numpy())
            a, bk, bv, _, _ = oracle.attention_bwd(qq.numpy(), kk.numpy(), vv.numpy(), gg.numpy(), causal, scale,
                                                   pos_q=_positions(q_range), pos_k=pk, lse=ll.numpy(), delta=delta,
                                                   nthreads=1)
            dq += torch.from_numpy(a)
            dk += torch.from_numpy(bk)   # the owner's accumulator, in shared memory
            dv += torch.from_numpy(bv)

        kv = ring_dist.PeerBlocks([kl.shape, vl.shape], kl.dtype, "cpu")
        acc = ring_dist.PeerBlocks([kl.shape, vl.shape], torch.float64, "cpu")
        kv.local[0].copy_(kl)
        kv.local[1].copy_(vl)
        want = oracle.attention_bwd(q, k, v, do, causal, 0.35, nthreads=1)[:3]
        errs = []
        for _ in range(2):                       # the accumulators reused by a second call
            seen.clear()
            dq, dk, dv = ring_dist.ring_attn_bwd_peer(ql, kv, ol, lsel, dol, layout, causal, 0.35, acc=acc,
                                                      compute=oracle_step)
            errs.append([float(np.max(np.abs(g.numpy() - w[:, pos]))) for g, w in zip((dq, dk, dv), want)])
        acc.close()
        kv.close()
        out[rank] = (errs, seen,
                     [int(oracle.layout.rank_positions(layout, world, S, (rank - s) % world)[0]) for s in range(world)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout,world,S,causal", [("zigzag", 2, 32, True), ("striped", 3, 24, True),
                                                   ("zigzag", 4, 64, True), ("contiguous", 3, 24, False)])
def test_peer_ring_backward_over_gloo_ranks(layout, world, S, causal):
    """The backward without sends (ring_attn_bwd_peer): step r adds rank i's shares for
    block (i - r) mod N into that block owner's dK, dV accumulators where they lie
    (shared memory on CPU ranks); the gradients of every rank equal the oracle's
    whole-sequence gradients, twice with the accumulators reused."""
    port = 29450 + (os.getpid() + world * 17 + S + int(causal)) % 900
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_peer_bwd_worker, args=(world, port, layout, S, causal, out), nprocs=world,
                       start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank, (errs, seen, want_seen) in out.items():
        for e in errs:
            assert max(e) <= 1e-9, (rank, errs)
        assert seen == want_seen, (rank, seen, want_seen)
