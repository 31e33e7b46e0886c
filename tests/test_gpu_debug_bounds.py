"""The bounds-checking build (libcpattn_debug.so, CP_DEBUG_BOUNDS=1): the tensor-core
kernels check every TMA coordinate and global index before the access and record a
failed check in the device status word instead of trapping (the stand-in for a
memory checker, which is closed on this machine).  A separate process loads that
build and runs the tensor-core paths on small and ragged shapes -- one-token,
odd-length and one-tile-plus-one sequences, N = 1, every layout, the stepwise ring
forms, the block and ring backward, the All-Gather forward and backward with
documents -- and each result must match the fp64 oracle with cp_stream_check
reporting no failed check."""
import os
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, out):
    os.environ["CP_LIBRARY"] = "debug"
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import cp_workloads as W
    import oracle
    import context_attention_cp_b200 as cp
    from gpu_helpers import np64
    assert cp.lib_path.endswith("libcpattn_debug.so")
    torch.cuda.set_device(0)
    errs = {}

    def ring(layout, N, S, causal, hq, hkv, mode):
        q, k, v = W.random_qkv(1, S, hq, hkv, 128, "bf16", seed=S + N)
        qr, kr, vr = (cp.layout_permute(t.cuda(), layout, N) for t in (q, k, v))
        o, lse = cp.ring_attn_fwd(qr, kr, vr, layout, N, causal, mode=mode)
        o = cp.layout_permute(o, layout, N, inverse=True)
        lse = cp.layout_permute(lse, layout, N, seq_axis=2, inverse=True)
        cp.stream_check()
        ro, rl = oracle.ring_attention(np64(q), np64(k), np64(v), layout, N, causal, 128 ** -0.5)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(np64(lse)), fin)
        return (float(np.max(np.abs(np64(o) - ro))), 2e-2), \
            (float(np.max(np.abs(np64(lse)[fin] - rl[fin]))) if fin.any() else 0.0, 1e-3)

    for case in [("contiguous", 1, 1, True, 2, 1, "fused"), ("contiguous", 1, 7, True, 2, 2, "fused"),
                 ("zigzag", 2, 260, True, 4, 1, "fused"), ("striped", 3, 387, True, 2, 1, "fused"),
                 ("contiguous", 2, 258, False, 2, 2, "fused"), ("zigzag", 4, 1032, True, 4, 2, "stepwise"),
                 ("striped", 4, 516, True, 4, 1, "stepwise_epi")]:
        errs["ring o %s" % (case,)], errs["ring lse %s" % (case,)] = ring(*case)

    # ring backward (tensor cores) on a ragged shape
    S, N = 520, 2
    q, k, v = W.random_qkv(1, S, 4, 1, 128, "bf16", seed=5)
    do = W.random_do(1, S, 4, 128, "bf16", seed=5)
    qr, kr, vr, dr = (cp.layout_permute(t.cuda(), "zigzag", N) for t in (q, k, v, do))
    o, lse = cp.ring_attn_fwd(qr, kr, vr, "zigzag", N, True)
    grads = cp.ring_attn_bwd(qr, kr, vr, o, lse, dr, "zigzag", N, True)
    grads = [cp.layout_permute(g, "zigzag", N, inverse=True) for g in grads]
    cp.stream_check()
    want = oracle.ring_attention_bwd(np64(q), np64(k), np64(v), np64(do), "zigzag", N, True, 128 ** -0.5)
    errs["ring bwd"] = (max(float(np.max(np.abs(np64(g) - w)) / np.max(np.abs(w))) for g, w in zip(grads, want)), 2e-2)

    # block backward (tensor cores, accumulating) with a ragged key block
    qb, kb, vb, dob = q[:, 200:412].contiguous(), k[:, :130].contiguous(), v[:, :130].contiguous(), \
        do[:, 200:412].contiguous()
    o_full, lse_full = oracle.attention(np64(q), np64(k), np64(v), True, 128 ** -0.5)
    ob = torch.from_numpy(o_full[:, 200:412]).to(torch.bfloat16)
    lb = torch.from_numpy(np.ascontiguousarray(lse_full[:, :, 200:412])).float()
    acc = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in (qb, kb, vb)]
    cp.block_attn_bwd(*(t.cuda() for t in (qb, kb, vb, ob, lb, dob)), ((200,), (212,), 1), ((0,), (130,), 1), True,
                      None, *acc)
    cp.stream_check()
    pq, pk = np.arange(200, 412), np.arange(130)
    delta = np.einsum("bshd,bshd->bhs", np64(dob), np64(ob))
    want = oracle.attention_bwd(np64(qb), np64(kb), np64(vb), np64(dob), True, 128 ** -0.5, pos_q=pq, pos_k=pk,
                                lse=np64(lb), delta=delta)[:3]
    errs["block bwd"] = (max(float(np.max(np.abs(np64(g) - w)) / np.max(np.abs(w))) for g, w in zip(acc, want)), 2e-2)

    # All-Gather with documents, forward and backward
    S, N, docs = 1032, 4, [0, 7, 300, 301, 777]
    q, k, v = W.random_qkv(1, S, 4, 1, 128, "bf16", seed=9)
    do = W.random_do(1, S, 4, 128, "bf16", seed=9)
    qr, kr, vr, dr = (cp.layout_permute(t.cuda(), "zigzag", N) for t in (q, k, v, do))
    o, lse = cp.allgather_attn_fwd(qr, kr, vr, "zigzag", N, True, docs)
    grads = cp.allgather_attn_bwd(qr, kr, vr, o, lse, dr, "zigzag", N, True, docs)
    o = cp.layout_permute(o, "zigzag", N, inverse=True)
    grads = [cp.layout_permute(g, "zigzag", N, inverse=True) for g in grads]
    cp.stream_check()
    ro, _ = oracle.attention_doc(np64(q), np64(k), np64(v), True, 128 ** -0.5, docs)
    errs["allgather fwd"] = (float(np.max(np.abs(np64(o) - ro))), 2e-2)
    want = oracle.attention_bwd_doc(np64(q), np64(k), np64(v), np64(do), True, 128 ** -0.5, docs)[:3]
    errs["allgather bwd"] = (max(float(np.max(np.abs(np64(g) - w)) / np.max(np.abs(w))) for g, w in zip(grads, want)),
                             2e-2)
    out["errs"] = errs


def test_debug_build_reports_no_bounds_failure():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.multiprocessing as mp
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(out,), nprocs=1, start_method="spawn", join=True)
    errs = out["errs"]
    assert len(errs) == 18
    for name, (e, bar) in errs.items():
        assert e <= bar, (name, e, bar)   # the bf16 bars: o 2e-2, lse 1e-3, gradients 2e-2 x max |reference|
