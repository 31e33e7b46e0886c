"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its own
timing, agree on the max over ranks (the time the whole-job throughput divides by),
and the reference arm runs on rank 0 only."""
import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.reduce_max(10.0 + 5.0 * rank, world, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = 29500 + os.getpid() % 1000
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_reduce_max_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1, "cpu") == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload = "fp32_s256_contig2"
        warmup = 1
        steps = 1
        gpus = 2
        ref_seconds = 0.1

    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    """Rank 0 prints one JSON line with the reference arm's keys: the oracle timed on
    host cores, e2e equal to the line's own value with no host-device bytes."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")

    class A:
        workload = "fp32_s256_contig2"
        warmup = 3
        steps = 1
        gpus = 1
        ref_seconds = 0.1

    assert bench.run_reference(A()) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["config"]["workload"] == "fp32_s256_contig2"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_appends_jsonl(monkeypatch, capsys, tmp_path):
    """--jsonl PATH appends the printed line to PATH, one record per run."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    path = tmp_path / "results.jsonl"

    class A:
        workload = "fp32_s256_contig2"
        warmup = 3
        steps = 1
        gpus = 1
        ref_seconds = 0.1
        jsonl = str(path)

    assert bench.run_reference(A()) == 0
    assert bench.run_reference(A()) == 0
    printed = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    stored = path.read_text().splitlines()
    assert len(stored) == 2 and stored == printed
    assert all(json.loads(ln)["impl"] == "reference" for ln in stored)


def _dist_worker(rank, world, port, out, ring="nccl"):
    """bench.run_dist on gloo ranks with the oracle as the block and merge steps."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK="0")
    import contextlib
    import io

    import numpy as np
    import torch

    import bench
    import oracle
    from test_ring_dist import _oracle_merge, _positions

    def step(qq, kk, vv, q_range, kv_range, causal, scale, o, lse, accumulate):
        scale = scale or qq.shape[-1] ** -0.5
        ob, lb = oracle.attention(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(), causal, scale,
                                  pos_q=_positions(q_range), pos_k=_positions(kv_range), nthreads=1)
        if accumulate:
            om, lm = oracle.lse_merge(o.double().numpy().transpose(0, 2, 1, 3), lse.double().numpy(),
                                      ob.transpose(0, 2, 1, 3), lb)
            ob, lb = om.transpose(0, 2, 1, 3), lm
        o.copy_(torch.from_numpy(np.ascontiguousarray(ob)))
        lse.copy_(torch.from_numpy(np.ascontiguousarray(lb)))

    class A:
        workload = "fp32_s256_contig2"
        warmup = 3
        steps = 2

    A.ring = ring
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_dist(A(), ring_kw={"compute": step, "merge": _oracle_merge}, device=torch.device("cpu"),
                            backend="gloo")
    out[rank] = (rc, buf.getvalue())


@pytest.mark.parametrize("ring", ["nccl", "peer"])
def test_run_dist_line_over_two_gloo_ranks(ring):
    """The --gpus N path of bench.py: every rank runs the real-rank ring on its block
    (blocks passed around, or read in place with --ring peer), the time is the max
    over ranks, and rank 0 alone prints one JSON line with the whole workload's
    throughput (strong scaling)."""
    import json
    port = 29550 + (os.getpid() + 3 * len(ring)) % 400
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_dist_worker, args=(2, port, out, ring), nprocs=2, start_method="spawn", join=True)
    assert out[0][0] == 0 and out[1][0] == 0
    assert out[1][1].strip() == ""
    lines = [ln for ln in out[0][1].splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["scaling"] == "strong" and d["value"] > 0
    assert d["config"]["workload"] == "fp32_s256_contig2" and d["config"]["N"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["value"] > 0
    assert d["config"]["ring"] == ring


def test_headline_traffic_comes_from_a_capture_of_the_current_kernel():
    """The bench line's roofline.traffic for the headline workload is read from the
    committed ncu summary, and only while the forward kernel's sources hash to the
    value recorded with the capture: a kernel change without a new capture reports
    null, and this test flags that the summary needs refreshing."""
    sys.path.insert(0, ROOT)
    import bench
    t = bench.profiled_traffic("llama3_70b_s128k_zigzag8")
    assert t is not None and t > 4.8e9      # at least Q + K + V + O once
    assert bench.profiled_traffic("no_such_workload") is None
