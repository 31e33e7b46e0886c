"""Benchmark: ring-attention forward TFLOP/s on effective (unmasked) FLOPs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mode fused|stepwise]
    python bench.py --impl reference ...     (the fp64 CPU oracle on a bounded row sample)

One step = one cp_ring_attn_fwd over the whole workload (all N virtual ranks, all
ring steps), inputs already permuted to rank-major order and resident in HBM.
The line also carries the standalone merge bandwidth, the backward
(cp_ring_attn_bwd) of the same workload and the All-Gather forward with a document
mask (cp_allgather_attn_fwd) on its 8-document variant, Ulysses
(cp_ulysses_attn_fwd, P = 4) on its shape and USP (cp_usp_attn_fwd: Ulysses groups
of 2 inside the workload's ring), each timed on its own.
L2 is flushed (a 256 MiB write) before every timed step; each step is timed with
CUDA events on the launching stream.  With --gpus N > 1 (torchrun) every rank
runs its own instance of the workload (weak scaling, no collective on the data
path); the time is the max over ranks.  Rank 0 prints one JSON line.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import cp_workloads as W  # noqa: E402

METRIC = "ring-attn fwd TFLOP/s (causal, effective FLOPs) & % bf16 peak; merge GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


KERNEL_SOURCES = ["context_attention_cp_b200/csrc/attn_tc.cu", "context_attention_cp_b200/csrc/ptx.cuh",
                  "context_attention_cp_b200/csrc/layout.h", "context_attention_cp_b200/csrc/kernels.h",
                  "context_attention_cp_b200/csrc/exp2_poly.h"]


def profiled_traffic(profile="profiles/attn_tc_kernel_llama3_8b_s8k_zigzag4.md"):
    """DRAM bytes per launch from the committed ncu summary, or None when the kernel
    sources changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, profile)) as f:
            text = f.read()
        h = hashlib.sha256()
        for name in KERNEL_SOURCES:
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    rec = dict(ln.split(":", 1) for ln in text.splitlines() if ln.startswith(("traffic_bytes_per_launch:",
                                                                              "source_sha256:")))
    if rec.get("source_sha256", "").strip() != h.hexdigest():
        return None
    return int(rec["traffic_bytes_per_launch"].strip())


def reduce_max(value, world, device):
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_rate(w, seconds_target=12.0, seed=0):
    """Times the fp64 oracle on a bounded sample of query rows of the workload.

    Returns (TFLOP/s on effective FLOPs, description, threads used).  The rows are
    exact answers (rows are independent), so the rate is the oracle's own."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(seed)
    q, k, v = W.make_inputs(w)
    k64 = k.float().numpy().astype(np.float64)
    v64 = v.float().numpy().astype(np.float64)
    threads = oracle.default_threads()

    def run(n):
        sel = np.stack([rng.integers(0, w.b, n), rng.integers(0, w.hq, n), rng.integers(0, w.S, n)], axis=1)
        q_sel = np.stack([q[b, p, h].float().numpy() for b, h, p in sel]).astype(np.float64)
        t0 = time.perf_counter()
        oracle.attention_rows(q_sel, sel, k64, v64, w.causal, w.scale, w.hq, nthreads=threads)
        dt = time.perf_counter() - t0
        pairs = sum((int(p) + 1) if w.causal else w.S for _, _, p in sel)
        return 4.0 * w.d * pairs / dt / 1e12, dt

    # grow the sample until one run takes about seconds_target
    n = threads
    rate, dt = run(n)
    while dt < 0.5 * seconds_target and n < 400000:
        n = min(400000, int(n * min(8.0, max(1.5, seconds_target / max(dt, 1e-3)))))
        rate, dt = run(n)
    return rate, "%d random query rows of %s (%.1f s of fp64 CPU work)" % (n, w.name, dt), threads


def run_reference(args):
    """The oracle as the reference arm, on the machine's host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.BY_NAME[args.workload]
    per = []
    desc = ""
    threads = 0
    # keep the whole run to a few minutes
    per_step = min(args.ref_seconds, 150.0 / (args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        rate, desc, threads = cpu_oracle_rate(w, seconds_target=per_step, seed=i)
        if i >= args.warmup:
            per.append(rate)
    value = statistics.mean(per)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "ms_per_step": None,
        "config": {"workload": w.name, "b": w.b, "S": w.S, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "layout": w.layout, "N": w.N, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.BENCH_WORKLOAD,
                    choices=sorted(n for n, x in W.BY_NAME.items() if x.n_docs == 1))
    ap.add_argument("--mode", default="fused", choices=["fused", "stepwise"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import context_attention_cp_b200 as cp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    w = W.BY_NAME[args.workload]
    peaks, peak_src = load_peaks()
    q, k, v = W.make_inputs(w)
    qd, kd, vd = (cp.layout_permute(t.to(dev), w.layout, w.N) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((w.b, w.hq, w.S), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ws_bytes = cp.ring_workspace_bytes(w.layout, w.N, args.mode, 0 if w.dtype == "bf16" else 1,
                                       w.b, w.S, w.hq, w.d)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        cp.ring_attn_fwd(qd, kd, vd, w.layout, w.N, w.causal, w.scale, o=o, lse=lse, mode=args.mode,
                         workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    cp.stream_check()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    cp.stream_check()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]  # ms
    total_ms = reduce_max(sum(times), world, dev)
    ms_per_step = total_ms / args.steps
    flops = w.effective_flops()
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12
    launches_per_step = 1 if (args.mode == "fused" or w.N == 1) else (2 * w.N - 1)

    # dominant kernel: the attention kernel (the whole fused ring is one launch)
    per_launch_tflops = flops / (ms_per_step * 1e-3) / 1e12 if args.mode == "fused" else None
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])

    # standalone merge bandwidth: one merge of a [b, S, Hq, d] fp32 accumulator with a
    # bf16 partial, bytes per (row, head) = (8 + 2) * d + 12; measured at this
    # workload's partial size and at the non-causal 64K workload's (16 heads), the
    # case with 31 merges per rank
    def merge_gbs(b, S, H, d):
        oa = torch.randn((b, S, H, d), device=dev)
        ob = torch.randn((b, S, H, d), device=dev).to(torch.bfloat16)
        la = torch.randn((b, H, S), device=dev)
        lb = torch.randn((b, H, S), device=dev)
        for _ in range(3):
            cp.lse_merge(oa, la, ob, lb)
        ms = []
        for _ in range(10):
            flush.zero_()
            m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            m0.record(stream)
            cp.lse_merge(oa, la, ob, lb)
            m1.record(stream)
            torch.cuda.synchronize()
            ms.append(m0.elapsed_time(m1))
        mbytes = b * S * H * ((8 + 2) * d + 12)
        t = statistics.mean(ms)
        gbs = mbytes / (t * 1e-3) / 1e9
        del oa, ob, la, lb
        return {"shape": [b, S, H, d], "gbs": gbs, "frac_of_measured_hbm": gbs / peaks.get("hbm_gbs", 6650.0),
                "frac_of_8tbs": gbs / 8000.0, "bytes_per_launch": mbytes, "ms_per_launch": t}

    merge = None
    if w.dtype == "bf16" and rank == 0:
        merge = merge_gbs(w.b, w.S, w.hq, w.d)
        w5 = W.BY_NAME["noncausal_s64k_contig32"]
        merge["noncausal_s64k_contig32"] = merge_gbs(w5.b, w5.S, w5.hq, w5.d)
        torch.cuda.empty_cache()

    # backward of the same workload (cp_ring_attn_bwd: statistics pass, the tcgen05
    # kernel, dq conversion), inputs resident, L2 flushed before every timed call;
    # effective FLOPs = 2.5x the forward's (five 2*d-flop products per visible pair)
    def bwd_leg():
        do = W.make_do(w).to(dev)
        dor = cp.layout_permute(do, w.layout, w.N)
        del do
        step()
        wsb = torch.empty(cp.ring_bwd_workspace_bytes(w.layout, w.N, 0, w.b, w.S, w.hq, w.d), dtype=torch.uint8,
                          device=dev)
        dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)

        def bstep():
            cp.ring_attn_bwd(qd, kd, vd, o, lse, dor, w.layout, w.N, w.causal, w.scale, dq, dk, dv, wsb)

        for _ in range(3):
            bstep()
        ms = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            bstep()
            b1.record(stream)
            torch.cuda.synchronize()
            ms.append(b0.elapsed_time(b1))
        cp.stream_check()
        t = statistics.mean(ms)
        tf = 2.5 * flops / (t * 1e-3) / 1e12
        del dor, wsb, dq, dk, dv
        torch.cuda.empty_cache()
        return {"metric": "ring-attn bwd TFLOP/s (effective: 5 products of 2*d flops per visible pair)",
                "value": tf, "unit": "TFLOP/s", "ms_per_step": t, "steps": len(ms), "launches_per_step": 3,
                "roofline": {"bound": "tensor", "kernel": "attn_bwd_kernel", "achieved": tf, "peak": peak_tf,
                             "unit": "TFLOP/s", "frac": tf / peak_tf, "peak_source": peak_src + " bf16 burst",
                             "timed": "whole call: statistics + attn_bwd_kernel + dq conversion",
                             "traffic": None}}

    backward = None
    if w.dtype == "bf16" and w.d == 128 and rank == 0:
        backward = bwd_leg()

    # All-Gather CP with a document mask (cp_allgather_attn_fwd: K and V gathered
    # into original order by two permute launches, then one document-masked pass),
    # on the 8-document variant of the 8B workload; effective FLOPs count only the
    # pairs the causal document mask leaves visible
    def allgather_leg():
        wd = W.BY_NAME["llama3_8b_s8k_zigzag4_docs8"]
        docs = wd.doc_starts()
        qa, ka, va = (cp.layout_permute(t.to(dev), wd.layout, wd.N) for t in W.make_inputs(wd))
        oa = torch.empty_like(qa)
        la = torch.empty((wd.b, wd.hq, wd.S), dtype=torch.float32, device=dev)
        wsa = torch.empty(cp.allgather_workspace_bytes(wd.N, 0, wd.b, wd.S, wd.hkv, wd.d, len(docs)),
                          dtype=torch.uint8, device=dev)

        def astep():
            cp.allgather_attn_fwd(qa, ka, va, wd.layout, wd.N, wd.causal, docs, wd.scale, oa, la, wsa)

        for _ in range(3):
            astep()
        ms = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            astep()
            a1.record(stream)
            torch.cuda.synchronize()
            ms.append(a0.elapsed_time(a1))
        cp.stream_check()
        t = statistics.mean(ms)
        tf = wd.effective_flops() / (t * 1e-3) / 1e12
        # its backward (gather, document-masked backward, dK/dV back to the ranks)
        doa = cp.layout_permute(W.random_do(wd.b, wd.S, wd.hq, wd.d, wd.dtype, wd.seed).to(dev), wd.layout, wd.N)
        gq, gk, gv = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
        wsb = torch.empty(cp.lib().cp_allgather_bwd_workspace_bytes(wd.N, 0, wd.b, wd.S, wd.hq, wd.hkv, wd.d, len(docs)),
                          dtype=torch.uint8, device=dev)

        def bstep():
            cp.allgather_attn_bwd(qa, ka, va, oa, la, doa, wd.layout, wd.N, wd.causal, docs, wd.scale, gq, gk, gv, wsb)

        for _ in range(3):
            bstep()
        bms = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            bstep()
            a1.record(stream)
            torch.cuda.synchronize()
            bms.append(a0.elapsed_time(a1))
        cp.stream_check()
        tb = statistics.mean(bms)
        tfb = 2.5 * wd.effective_flops() / (tb * 1e-3) / 1e12
        del qa, ka, va, oa, la, wsa, doa, gq, gk, gv, wsb
        torch.cuda.empty_cache()
        return {"metric": "all-gather CP fwd TFLOP/s (causal document mask, effective FLOPs)", "workload": wd.name,
                "backward": {"value": tfb, "unit": "TFLOP/s", "ms_per_step": tb, "frac": tfb / peak_tf,
                             "launches_per_step": 7,
                             "timed": "K, V gather + statistics + backward kernel + dq conversion + dK, dV scatter"},
                "n_docs": len(docs), "value": tf, "unit": "TFLOP/s", "ms_per_step": t, "steps": len(ms),
                "launches_per_step": 3,
                "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (document variant)", "achieved": tf,
                             "peak": peak_tf, "unit": "TFLOP/s", "frac": tf / peak_tf,
                             "peak_source": peak_src + " bf16 burst",
                             "timed": "whole call: K and V gather + document-masked attention", "traffic": None}}

    allgather = None
    if w.dtype == "bf16" and w.d == 128 and rank == 0:
        allgather = allgather_leg()

    # Ulysses over P = 4 virtual ranks on this workload's shape (original order):
    # all-to-all of q, k, v, one attention launch over the head groups, all-to-all
    # of o and lse back (5 + 1 launches)
    def ulysses_leg(P=4, usp=False):
        # usp: Ulysses groups of P inside each of the workload's N ring groups (the
        # inputs in the ring's rank-major order, permuted before the timed region)
        qu, ku, vu = (t.to(dev) for t in W.make_inputs(w))
        if usp:
            qu, ku, vu = (cp.layout_permute(t, w.layout, w.N) for t in (qu, ku, vu))
        ou = torch.empty_like(qu)
        lu = torch.empty((w.b, w.hq, w.S), dtype=torch.float32, device=dev)
        wsu = torch.empty(cp.ulysses_workspace_bytes(P, 0, w.b, w.S, w.hq, w.hkv, w.d), dtype=torch.uint8, device=dev)

        def ustep():
            if usp:
                cp.usp_attn_fwd(qu, ku, vu, w.layout, w.N, P, w.causal, w.scale, ou, lu, wsu)
            else:
                cp.ulysses_attn_fwd(qu, ku, vu, P, w.causal, w.scale, ou, lu, wsu)

        for _ in range(3):
            ustep()
        ms = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            u0.record(stream)
            ustep()
            u1.record(stream)
            torch.cuda.synchronize()
            ms.append(u0.elapsed_time(u1))
        cp.stream_check()
        t = statistics.mean(ms)
        tf = flops / (t * 1e-3) / 1e12
        del qu, ku, vu, ou, lu, wsu
        torch.cuda.empty_cache()
        return {"metric": ("USP" if usp else "Ulysses") + " fwd TFLOP/s (causal, effective FLOPs)", "P": P,
                "ring": {"layout": w.layout, "N": w.N} if usp else None, "value": tf, "unit": "TFLOP/s",
                "ms_per_step": t, "steps": len(ms), "launches_per_step": 6,
                "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": tf, "peak": peak_tf,
                             "unit": "TFLOP/s", "frac": tf / peak_tf, "peak_source": peak_src + " bf16 burst",
                             "timed": "whole call: 5 all-to-all launches + attention", "traffic": None}}

    ulysses = None
    if w.dtype == "bf16" and w.hkv % 4 == 0 and w.hq % 4 == 0 and w.S % 4 == 0 and rank == 0:
        ulysses = ulysses_leg()
        if w.hkv % 2 == 0 and w.S % (2 * w.N) == 0:
            ulysses["usp"] = ulysses_leg(P=2, usp=True)

    # end to end through the public API, every step: pinned host -> device copy of
    # q/k/v, permute to rank-major order, ring attention, unpermute, device -> host
    # copy of o and lse.  Consecutive steps are pipelined on three streams (copy-in,
    # compute, copy-out) with double-buffered device tensors, as a serving loop would
    # run them; the time runs from the first copy-in to the last copy-out.
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lh = torch.empty((w.b, w.hq, w.S), dtype=torch.float32).pin_memory()
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    buf_in = [[torch.empty_like(t, device=dev) for t in (q, k, v)] for _ in range(2)]
    buf_out = [(torch.empty(q.shape, dtype=q.dtype, device=dev),
                torch.empty((w.b, w.hq, w.S), dtype=torch.float32, device=dev)) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        sl = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[sl])  # step i-2 finished reading these inputs
            for src, dst in zip((qh, kh, vh), buf_in[sl]):
                dst.copy_(src, non_blocking=True)
            ev_in[sl].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[sl])
            s_cmp.wait_event(ev_out[sl])  # step i-2's outputs have left the device
            qr, kr, vr = (cp.layout_permute(t, w.layout, w.N) for t in buf_in[sl])
            og, lg = cp.ring_attn_fwd(qr, kr, vr, w.layout, w.N, w.causal, w.scale, mode=args.mode, workspace=ws)
            cp.layout_permute(og, w.layout, w.N, inverse=True, out=buf_out[sl][0])
            cp.layout_permute(lg, w.layout, w.N, seq_axis=2, inverse=True, out=buf_out[sl][1])
            ev_cmp[sl].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[sl])
            oh.copy_(buf_out[sl][0], non_blocking=True)
            lh.copy_(buf_out[sl][1], non_blocking=True)
            ev_out[sl].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(e_steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    cp.stream_check()
    e_ms = reduce_max(e0.elapsed_time(e1), world, dev)
    e2e_value = world * flops * e_steps / (e_ms * 1e-3) / 1e12
    es = 2 if w.dtype == "bf16" else 4
    h2d = (q.numel() + k.numel() + v.numel()) * es
    d2h = q.numel() * es + w.b * w.hq * w.S * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, threads = cpu_oracle_rate(w)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "b": w.b, "S": w.S, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                       "layout": w.layout, "N": w.N, "causal": w.causal, "mode": args.mode,
                       "l2": "flushed before every timed step (256 MiB write)",
                       "parallelism": "replicas x%d" % world},
            "pct_bf16_peak": value / world / peak_tf,
            "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel",
                         "achieved": per_launch_tflops, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": (per_launch_tflops / peak_tf) if per_launch_tflops else None,
                         "peak_source": peak_src + " bf16 burst",
                         "traffic": profiled_traffic() if w.name == W.BENCH_WORKLOAD else None},
            "merge": merge,
            "backward": backward,
            "allgather": allgather,
            "ulysses": ulysses,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e_ms / e_steps, "pipelined": "copy-in / compute / copy-out on 3 streams"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
