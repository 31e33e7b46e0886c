"""Benchmark: ring-attention forward TFLOP/s on effective (unmasked) FLOPs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mode M] [--legs L]
    python bench.py --impl reference ...     (the fp64 CPU oracle on a bounded row sample)

Headline (one GPU): one step = one cp_ring_attn_fwd over the whole workload (all N
virtual ranks, all ring steps), inputs already permuted to rank-major order and
resident in HBM.  The default workload is the largest one that fits one GPU: the
Llama-3-70B head shape (64 query / 8 KV heads, d = 128) at S = 131072, causal,
zig-zag over N = 8 virtual ranks.

The same line carries, each timed on its own (CUDA events on the launching stream,
L2 flushed before every timed call):
  configs   : the other bf16 workloads (fused ring), and the two stepwise forms of
              the ring (block launches + standalone merges, the page's loop as
              written; block launches merging in their epilogue) on the 8B and the
              non-causal 64K workloads, with the standalone merge's share;
  merge     : the standalone LSE merge's HBM bandwidth at two partial sizes, and
              the layout permute's on this workload's q, k and lse;
  backward  : cp_ring_attn_bwd on the headline workload and the 8B one;
  allgather : All-Gather CP with a document mask (8 and 32 documents), forward and
              backward;
  ulysses   : Ulysses (P = 4) and USP (Ulysses groups of 2 inside the ring);
  e2e       : the headline through the public API with host buffers (pinned
              host -> device copies of q, k, v, permute, ring, unpermute, device ->
              host copies of o and lse), pipelined on three streams;
  cpu_baseline : the fp64 oracle on the host cores, on a bounded row sample.

With --gpus N > 1 (torchrun, one process per GPU) the ring runs across the N real
ranks instead (context_attention_cp_b200.ring_dist): each rank holds its layout
block of the workload (c = S / N tokens) and passes K/V blocks to its neighbour
with NCCL point-to-point transfers while its block kernel runs; with --ring peer
the blocks stay where they are and each step's block kernel reads the other rank's
K/V from its memory (ring_dist.ring_attn_fwd_peer).  The total work is the
workload's, whatever N (strong scaling); the time is the max over ranks.
Rank 0 prints one JSON line.
"""
import argparse
import hashlib
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
VENDOR_BF16_DENSE_TFLOPS = 2250.0   # B200 dense bf16 (the 2:4-sparse figure halved)
L2_FLUSH_BYTES = 256 << 20
# GPU-side delay (clock cycles, about 0.2 ms) queued after the L2 flush and before a
# start event: the host marshals the call's arguments while the GPU is still busy, so
# the start event fires when the GPU reaches the call and the timed region holds the
# call's device work only (the host's per-call cost is in the end-to-end figure).
HOLD_CYCLES = 400_000


def emit(line, args):
    """Prints the JSON line; with --jsonl PATH also appends it to PATH (one record per
    line, for keeping results across runs)."""
    text = json.dumps(line)
    print(text, flush=True)
    path = getattr(args, "jsonl", None)
    if path:
        with open(path, "a") as f:
            f.write(text + "\n")


class L2Flush:
    """Empties the L2 of the timed call's data before each timed call.

    A 256 MiB write evicts everything the call could find in the 126 MB L2, but it
    leaves the L2 full of dirty lines, and their write-back to HBM would land inside
    the next timed region (about 20 us of DRAM time: as long as a whole merge or lse
    permute launch).  A read of a second 256 MiB buffer follows, so the timed call
    starts from an L2 of clean, unrelated lines, as under the profiler's cache
    control.  Then the GPU-side hold (HOLD_CYCLES)."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()
        self.torch.cuda._sleep(HOLD_CYCLES)


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


def kernel_source_sha():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload):
    """DRAM bytes per launch of the forward kernel on `workload`, from the committed
    ncu summary profiles/attn_tc_kernel_<workload>.md; None when there is none or
    when the kernel sources changed since its counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "attn_tc_kernel_%s.md" % workload)) as f:
            text = f.read()
        sha = kernel_source_sha()
    except OSError:
        return None
    rec = dict(ln.split(":", 1) for ln in text.splitlines() if ln.startswith(("traffic_bytes_per_launch:",
                                                                              "source_sha256:")))
    if rec.get("source_sha256", "").strip() != sha or "traffic_bytes_per_launch" not in rec:
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


def cpu_oracle_rate(w, seconds_target=12.0, seed=0, threads=None, inputs=None):
    """Times the fp64 oracle on a bounded sample of query rows of the workload.

    Returns (TFLOP/s on effective FLOPs, description, threads used).  The rows are
    exact answers (rows are independent), so the rate is the oracle's own."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(seed)
    q, k, v = inputs if inputs is not None else W.make_inputs(w)
    k64 = k.float().numpy().astype(np.float64)
    v64 = v.float().numpy().astype(np.float64)
    if threads is None:
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
    inputs = W.make_inputs(w)
    for i in range(args.warmup + args.steps):
        rate, desc, threads = cpu_oracle_rate(w, seconds_target=per_step, seed=i, inputs=inputs)
        if i >= args.warmup:
            per.append(rate)
    value = statistics.mean(per)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        # a whole step (every query row) is never run: the time one would take at the
        # sampled rate
        "ms_per_step": w.effective_flops() / (value * 1e12) * 1e3 if value > 0 else None,
        "ms_per_step_how": "extrapolated: the workload's effective FLOPs / the sampled rate",
        "config": {"workload": w.name, "b": w.b, "S": w.S, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "layout": w.layout, "N": w.N, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, args)
    return 0


class Timer:
    """CUDA-event timing of calls on the current stream, L2 flushed before each."""

    def __init__(self, torch, flush):
        self.torch = torch
        self.flush = flush

    def __call__(self, fn, steps, warmup=3):
        torch = self.torch
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            fn()
        ms = []
        for _ in range(steps):
            self.flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.mean(ms), ms


def tflops_entry(flops, ms, peak_tf, peak_src, **extra):
    tf = flops / (ms * 1e-3) / 1e12
    d = {"value": tf, "unit": "TFLOP/s", "ms_per_step": ms, "frac": tf / peak_tf,
         "frac_of": "%s bf16 burst %.1f TFLOP/s" % (peak_src, peak_tf)}
    d.update(extra)
    return d


def run_legs(cp, torch, dev, w, qd, kd, vd, o, lse, timer, peaks, peak_src, args, legs):
    """The sub-results of the one-GPU line (see the module docstring)."""
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    steps = max(3, min(args.steps, 10))
    out = {}

    def merge_gbs(b, S, H, d):
        oa = torch.randn((b, S, H, d), device=dev)
        ob = torch.randn((b, S, H, d), device=dev).to(torch.bfloat16)
        la = torch.randn((b, H, S), device=dev)
        lb = torch.randn((b, H, S), device=dev)
        t, _ = timer(lambda: cp.lse_merge(oa, la, ob, lb), steps)
        mbytes = b * S * H * ((8 + 2) * d + 12)
        gbs = mbytes / (t * 1e-3) / 1e9
        del oa, ob, la, lb
        torch.cuda.empty_cache()
        return {"shape": [b, S, H, d], "gbs": gbs, "frac_of_measured_hbm": gbs / hbm, "frac_of_8tbs": gbs / 8000.0,
                "bytes_per_launch": mbytes, "ms_per_launch": t}

    def permute_gbs(x, seq_axis=1, inverse=False):
        y = torch.empty_like(x)
        t, ms = timer(lambda: cp.layout_permute(x, w.layout, w.N, seq_axis=seq_axis, inverse=inverse, out=y), steps)
        nbytes = 2 * x.numel() * x.element_size()
        gbs = nbytes / (t * 1e-3) / 1e9
        del y
        torch.cuda.empty_cache()
        return {"shape": list(x.shape), "seq_axis": seq_axis, "inverse": inverse, "gbs": gbs,
                "frac_of_measured_hbm": gbs / hbm, "bytes_per_launch": nbytes, "ms_per_launch": t,
                "ms_median": statistics.median(ms)}

    if "merge" in legs:
        w2, w5 = W.BY_NAME["llama3_8b_s8k_zigzag4"], W.BY_NAME["noncausal_s64k_contig32"]
        out["merge"] = {w2.name: merge_gbs(w2.b, w2.S, w2.hq, w2.d), w5.name: merge_gbs(w5.b, w5.S, w5.hq, w5.d)}
        # the layout permute on this workload's tensors: bytes = read + write of the tensor
        out["permute"] = {"layout": w.layout, "n_ranks": w.N,
                          "q": permute_gbs(qd), "o_inverse": permute_gbs(qd, inverse=True),
                          "k": permute_gbs(kd), "lse_inverse": permute_gbs(lse, seq_axis=2, inverse=True)}

    if "configs" in legs:
        cfgs = {}
        for wx in W.WORKLOADS:
            if wx.dtype != "bf16" or wx.n_docs != 1:
                continue
            same = wx.name == w.name
            if same:
                qx, kx, vx, ox, lx = qd, kd, vd, o, lse
            else:
                qx, kx, vx = (cp.layout_permute(t.to(dev), wx.layout, wx.N) for t in W.make_inputs(wx))
                ox = torch.empty_like(qx)
                lx = torch.empty((wx.b, wx.hq, wx.S), dtype=torch.float32, device=dev)
            flops = wx.effective_flops()
            ent = {}
            modes = ["fused"] if not same else []
            if wx.name in ("llama3_8b_s8k_zigzag4", "noncausal_s64k_contig32") or same:
                modes += ["stepwise", "stepwise_epi"]
            for mode in modes:
                need = cp.ring_workspace_bytes(wx.layout, wx.N, mode, 0, wx.b, wx.S, wx.hq, wx.d)
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
                st = 3 if same else steps
                t, _ = timer(lambda: cp.ring_attn_fwd(qx, kx, vx, wx.layout, wx.N, wx.causal, o=ox, lse=lx, mode=mode,
                                                      workspace=ws), st)
                e = tflops_entry(flops, t, peak_tf, peak_src,
                                 launches_per_step=1 if mode == "fused" else (wx.N if mode == "stepwise_epi"
                                                                              else 2 * wx.N - 1))
                if mode == "stepwise":
                    # share of the N - 1 standalone merges, from one merge timed alone at this size
                    oa = torch.empty((wx.b, wx.S, wx.hq, wx.d), dtype=torch.float32, device=dev)
                    ob = torch.empty((wx.b, wx.S, wx.hq, wx.d), dtype=torch.bfloat16, device=dev)
                    la = torch.zeros((wx.b, wx.hq, wx.S), dtype=torch.float32, device=dev)
                    lb = torch.zeros((wx.b, wx.hq, wx.S), dtype=torch.float32, device=dev)
                    tm, _ = timer(lambda: cp.lse_merge(oa, la, ob, lb), steps)
                    mb = wx.b * wx.S * wx.hq * ((8 + 2) * wx.d + 12)
                    e["merge"] = {"ms_per_merge": tm, "merges_per_step": wx.N - 1,
                                  "share_of_step": (wx.N - 1) * tm / t, "gbs": mb / (tm * 1e-3) / 1e9,
                                  "how": "one standalone merge of this size timed alone, times N - 1"}
                    del oa, ob, la, lb
                ent[mode] = e
                del ws
            cfgs[wx.name] = ent
            if not same:
                del qx, kx, vx, ox, lx
            torch.cuda.empty_cache()
        out["configs"] = cfgs

    def bwd(wx, qx, kx, vx, ox, lx, n_steps):
        dor = cp.layout_permute(W.make_do(wx).to(dev), wx.layout, wx.N)
        cp.ring_attn_fwd(qx, kx, vx, wx.layout, wx.N, wx.causal, o=ox, lse=lx)
        wsb = torch.empty(cp.ring_bwd_workspace_bytes(wx.layout, wx.N, 0, wx.b, wx.S, wx.hq, wx.d),
                          dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(qx), torch.empty_like(kx), torch.empty_like(vx)
        t, _ = timer(lambda: cp.ring_attn_bwd(qx, kx, vx, ox, lx, dor, wx.layout, wx.N, wx.causal, None, dq, dk, dv,
                                              wsb), n_steps)
        cp.stream_check()
        del dor, wsb, dq, dk, dv
        torch.cuda.empty_cache()
        return tflops_entry(2.5 * wx.effective_flops(), t, peak_tf, peak_src, launches_per_step=3,
                            kernel="attn_bwd_kernel",
                            timed="whole call: statistics + attn_bwd_kernel + dq conversion")

    if "backward" in legs and w.dtype == "bf16" and w.d == 128:
        b = {"metric": "ring-attn bwd TFLOP/s (effective: 5 products of 2*d flops per visible pair)"}
        b[w.name] = bwd(w, qd, kd, vd, o, lse, 3)
        w2 = W.BY_NAME["llama3_8b_s8k_zigzag4"]
        if w2.name != w.name:
            q2, k2, v2 = (cp.layout_permute(t.to(dev), w2.layout, w2.N) for t in W.make_inputs(w2))
            o2, l2 = torch.empty_like(q2), torch.empty((w2.b, w2.hq, w2.S), dtype=torch.float32, device=dev)
            b[w2.name] = bwd(w2, q2, k2, v2, o2, l2, steps)
            del q2, k2, v2, o2, l2
            torch.cuda.empty_cache()
        out["backward"] = b

    if "allgather" in legs:
        ag = {"metric": "all-gather CP TFLOP/s (causal document mask, effective FLOPs)"}
        for name in ("llama3_8b_s8k_zigzag4_docs8", "llama3_8b_s8k_zigzag4_docs32"):
            wd = W.BY_NAME[name]
            docs = wd.doc_starts()
            qa, ka, va = (cp.layout_permute(t.to(dev), wd.layout, wd.N) for t in W.make_inputs(wd))
            oa = torch.empty_like(qa)
            la = torch.empty((wd.b, wd.hq, wd.S), dtype=torch.float32, device=dev)
            wsa = torch.empty(cp.allgather_workspace_bytes(wd.N, 0, wd.b, wd.S, wd.hkv, wd.d, len(docs)),
                              dtype=torch.uint8, device=dev)
            t, _ = timer(lambda: cp.allgather_attn_fwd(qa, ka, va, wd.layout, wd.N, wd.causal, docs, None, oa, la,
                                                       wsa), steps)
            cp.stream_check()
            # the library reads the ranks' K/V blocks in place when every key tile is a run
            # of consecutive rank-major rows (contiguous; zig-zag chunks of whole tiles)
            c = wd.S // wd.N
            in_place = wd.dtype == "bf16" and (wd.layout == "contiguous" or
                                               (wd.layout == "zigzag" and (c // 2) % 128 == 0))
            gather = "" if in_place else "K and V gather + "
            e = {"n_docs": len(docs),
                 "forward": tflops_entry(wd.effective_flops(), t, peak_tf, peak_src,
                                         launches_per_step=2 if in_place else 4,
                                         kernel="attn_tc_kernel (document variant)",
                                         timed="whole call: " + gather + "document tables + document-masked"
                                               " attention" + (" (K/V read in place)" if in_place else ""))}
            doa = cp.layout_permute(W.make_do(wd).to(dev), wd.layout, wd.N)
            gq, gk, gv = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
            wsb = torch.empty(cp.lib().cp_allgather_bwd_workspace_bytes(wd.N, 0, wd.b, wd.S, wd.hq, wd.hkv, wd.d,
                                                                        len(docs)), dtype=torch.uint8, device=dev)
            tb, _ = timer(lambda: cp.allgather_attn_bwd(qa, ka, va, oa, la, doa, wd.layout, wd.N, wd.causal, docs,
                                                        None, gq, gk, gv, wsb), steps)
            cp.stream_check()
            e["backward"] = tflops_entry(2.5 * wd.effective_flops(), tb, peak_tf, peak_src,
                                         launches_per_step=4 if in_place else 8,
                                         timed="whole call: " + gather + "document tables + statistics + backward"
                                               " kernel + dq conversion" + ("" if in_place else " + dK, dV scatter"))
            ag[name] = e
            del qa, ka, va, oa, la, wsa, doa, gq, gk, gv, wsb
            torch.cuda.empty_cache()
        out["allgather"] = ag

    if "ulysses" in legs:
        w2 = W.BY_NAME["llama3_8b_s8k_zigzag4"]

        def uly(P, usp):
            qu, ku, vu = (t.to(dev) for t in W.make_inputs(w2))
            if usp:
                qu, ku, vu = (cp.layout_permute(t, w2.layout, w2.N) for t in (qu, ku, vu))
            ou = torch.empty_like(qu)
            lu = torch.empty((w2.b, w2.hq, w2.S), dtype=torch.float32, device=dev)
            wsu = torch.empty(cp.ulysses_workspace_bytes(P, 0, w2.b, w2.S, w2.hq, w2.hkv, w2.d), dtype=torch.uint8,
                              device=dev)
            if usp:
                fn = lambda: cp.usp_attn_fwd(qu, ku, vu, w2.layout, w2.N, P, w2.causal, None, ou, lu, wsu)  # noqa
            else:
                fn = lambda: cp.ulysses_attn_fwd(qu, ku, vu, P, w2.causal, None, ou, lu, wsu)  # noqa
            t, _ = timer(fn, steps)
            cp.stream_check()
            del qu, ku, vu, ou, lu, wsu
            torch.cuda.empty_cache()
            return tflops_entry(w2.effective_flops(), t, peak_tf, peak_src, P=P, launches_per_step=6,
                                ring={"layout": w2.layout, "N": w2.N} if usp else None,
                                timed="whole call: 5 all-to-all launches + attention")

        out["ulysses"] = {"workload": w2.name, "ulysses_P4": uly(4, False), "usp_P2": uly(2, True)}
    return out


def cpu_baseline(w, inputs):
    """The oracle on all host threads and on one, with the full run extrapolated."""
    import oracle
    rate, desc, threads = cpu_oracle_rate(w, inputs=inputs)
    rate1, desc1, _ = cpu_oracle_rate(w, seconds_target=8.0, seed=1, threads=1, inputs=inputs)
    full = w.effective_flops()
    return {"value": rate, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
            "single_thread": {"value": rate1, "unit": "TFLOP/s", "cores": 1, "sample": desc1},
            "full_run_s_extrapolated": {"all_threads": full / (rate * 1e12), "single_thread": full / (rate1 * 1e12),
                                        "how": "extrapolated: the workload's effective FLOPs / the sampled rate"},
            "host_threads_available": len(os.sched_getaffinity(0)), "oracle_default_threads": oracle.default_threads()}


def run_one_gpu(args):
    import torch

    import context_attention_cp_b200 as cp

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = W.BY_NAME[args.workload]
    peaks, peak_src = load_peaks()
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    inputs = W.make_inputs(w)
    q, k, v = inputs
    qd, kd, vd = (cp.layout_permute(t.to(dev), w.layout, w.N) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((w.b, w.hq, w.S), dtype=torch.float32, device=dev)
    flush = L2Flush(torch, dev)
    ws_bytes = cp.ring_workspace_bytes(w.layout, w.N, args.mode, 0 if w.dtype == "bf16" else 1, w.b, w.S, w.hq, w.d)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        cp.ring_attn_fwd(qd, kd, vd, w.layout, w.N, w.causal, o=o, lse=lse, mode=args.mode, workspace=ws)

    for _ in range(args.warmup):
        flush()
        step()
    cp.stream_check()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    cp.stream_check()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]  # ms
    total_ms = sum(times)
    ms_per_step = total_ms / args.steps
    flops = w.effective_flops()
    value = flops * args.steps / (total_ms * 1e-3) / 1e12
    launches_per_step = {"fused": 1, "stepwise": 2 * w.N - 1, "stepwise_epi": w.N}[args.mode] if w.N > 1 else 1

    legs = set(args.legs.split(",")) if args.legs not in ("all", "none") else (
        {"merge", "configs", "backward", "allgather", "ulysses"} if args.legs == "all" else set())
    timer = Timer(torch, flush)
    extra = run_legs(cp, torch, dev, w, qd, kd, vd, o, lse, timer, peaks, peak_src, args, legs) if legs else {}

    # end to end through the public API, every step: pinned host -> device copy of
    # q/k/v, permute to rank-major order, ring attention, unpermute, device -> host
    # copy of o and lse.  Consecutive steps are pipelined on three streams (copy-in,
    # compute, copy-out) with double-buffered device tensors, as a serving loop would
    # run them; the time runs from the first copy-in to the last copy-out.
    del flush
    torch.cuda.empty_cache()
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
            og, lg = cp.ring_attn_fwd(qr, kr, vr, w.layout, w.N, w.causal, mode=args.mode, workspace=ws)
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
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(e_steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    cp.stream_check()
    e_ms = e0.elapsed_time(e1)
    e2e_value = flops * e_steps / (e_ms * 1e-3) / 1e12
    es = 2 if w.dtype == "bf16" else 4
    h2d = (q.numel() + k.numel() + v.numel()) * es
    d2h = q.numel() * es + w.b * w.hq * w.S * 4
    del buf_in, buf_out, qh, kh, vh, oh, lh

    cpu = None if args.no_cpu_baseline else cpu_baseline(w, inputs)
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step,
        "step_ms": {"median": statistics.median(times), "best": min(times), "worst": max(times)},
        "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "b": w.b, "S": w.S, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "layout": w.layout, "N": w.N, "causal": w.causal, "mode": args.mode,
                   "l2": "flushed before every timed step (256 MiB write, then a 256 MiB read so no dirty line is left);"
                         " inputs also exceed L2",
                   "parallelism": "one GPU, %d virtual ranks" % w.N},
        "pct_bf16_peak": value / peak_tf,
        "pct_vendor_bf16_dense": value / VENDOR_BF16_DENSE_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel" if args.mode == "fused" or w.dtype == "bf16"
                     else "attn_simt_kernel",
                     "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                     "peak_source": peak_src + " bf16 burst",
                     "secondary": {"peak": VENDOR_BF16_DENSE_TFLOPS, "frac": achieved / VENDOR_BF16_DENSE_TFLOPS,
                                   "source": "vendor dense bf16 (2:4-sparse figure halved)"},
                     "sustained": {"peak": peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]),
                                   "frac": achieved / peaks.get("bf16_tflops_sustained",
                                                                FALLBACK_PEAKS["bf16_tflops_sustained"]),
                                   "source": peak_src + " bf16 sustained (seconds of back-to-back GEMMs under the power"
                                             " cap)", "timed_region_s": total_ms / 1e3,
                                   "power_capped": bool(clk and "sw_power_cap" in clk.get("reasons", []))},
                     "timed": "whole call (one launch in fused mode), CUDA events on the launching stream",
                     "traffic": profiled_traffic(w.name) if args.mode == "fused" else None},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms / e_steps, "pipelined": "copy-in / compute / copy-out on 3 streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    line.update(extra)
    emit(line, args)
    return 0


def dist_inputs(w, rank, world, dev, torch):
    """This rank's layout block of the workload (c = S / world tokens), drawn on the
    device from a generator seeded with the workload's seed and the rank (every
    rank draws only its own tokens)."""
    c = w.S // world
    g = torch.Generator(device=dev).manual_seed(w.seed * 1000 + rank)
    td = W.torch_dtype(w.dtype)
    q = torch.randn((w.b, c, w.hq, w.d), generator=g, device=dev, dtype=torch.float32).to(td)
    k = torch.randn((w.b, c, w.hkv, w.d), generator=g, device=dev, dtype=torch.float32).to(td)
    v = torch.randn((w.b, c, w.hkv, w.d), generator=g, device=dev, dtype=torch.float32).to(td)
    if w.k_scale != 1.0:
        k = k * w.k_scale
    return q, k, v


def run_dist(args, ring_kw=None, device=None, backend="nccl"):
    """The ring across real ranks: one process per GPU (see the module docstring).

    ring_kw / device / backend exist for the CPU test of this plumbing (gloo ranks,
    injected block and merge steps); the bench itself uses the defaults."""
    import datetime

    import torch
    import torch.distributed as dist

    from context_attention_cp_b200 import ring_dist

    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if device is None:
        torch.cuda.set_device(local)
        device = torch.device("cuda", local)
    cuda = device.type == "cuda"
    w = W.BY_NAME[args.workload]
    if w.S % world or (w.layout == "zigzag" and w.S % (2 * world)):
        raise SystemExit("the workload's S does not split over %d ranks" % world)
    peaks, peak_src = load_peaks()
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    q, k, v = dist_inputs(w, rank, world, device, torch)
    kw = dict(ring_kw or {})
    ring = getattr(args, "ring", "nccl")
    kv = None
    if ring == "peer":
        # every rank maps the others' K/V blocks once; the block kernels read them in place
        kv = ring_dist.PeerBlocks([k.shape, v.shape], k.dtype, device)
        kv.local[0].copy_(k)
        kv.local[1].copy_(v)

    def step():
        if kv is not None:
            return ring_dist.ring_attn_fwd_peer(q, kv, w.layout, w.causal, **kw)
        return ring_dist.ring_attn_fwd_dist(q, k, v, w.layout, w.causal, **kw)

    for _ in range(args.warmup):
        step()
    if cuda:
        torch.cuda.synchronize()
    dist.barrier()
    clocks = ClockSampler(local) if (cuda and rank == 0) else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if cuda:
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    if cuda:
        e1.record()
        torch.cuda.synchronize()
        my_ms = e0.elapsed_time(e1)
    else:
        my_ms = (time.perf_counter() - t0) * 1e3
    dist.barrier()
    clk = clocks.stop() if clocks else None
    total_ms = reduce_max(my_ms, world, device)
    ms_per_step = total_ms / args.steps
    flops = w.effective_flops()
    value = flops * args.steps / (total_ms * 1e-3) / 1e12

    # end to end: this rank's inputs from pinned host memory, the ring, o and lse back
    qh, kh, vh = (t.cpu() for t in (q, k, v))
    if cuda:
        qh, kh, vh = (t.pin_memory() for t in (qh, kh, vh))
    e_steps = max(3, min(args.steps, 5))
    dist.barrier()
    t1 = time.perf_counter()
    if cuda:
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
    for _ in range(e_steps):
        qx = qh.to(device, non_blocking=True)
        if kv is not None:
            kv.local[0].copy_(kh, non_blocking=True)
            kv.local[1].copy_(vh, non_blocking=True)
            ox, lx = ring_dist.ring_attn_fwd_peer(qx, kv, w.layout, w.causal, **kw)
        else:
            kx, vx = (t.to(device, non_blocking=True) for t in (kh, vh))
            ox, lx = ring_dist.ring_attn_fwd_dist(qx, kx, vx, w.layout, w.causal, **kw)
        ox.cpu(), lx.cpu()
    if cuda:
        f1.record()
        torch.cuda.synchronize()
        e_my = f0.elapsed_time(f1)
    else:
        e_my = (time.perf_counter() - t1) * 1e3
    e_ms = reduce_max(e_my, world, device)
    if kv is not None:
        kv.close()
    es = 2 if w.dtype == "bf16" else 4
    h2d = world * (q.numel() + k.numel() + v.numel()) * es
    d2h = world * (q.numel() * es + w.b * w.hq * (w.S // world) * 4)
    dist.barrier()
    if rank == 0:
        per_gpu = value / world
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (per-rank device generator)",
            "config": {"workload": w.name, "b": w.b, "S": w.S, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                       "layout": w.layout, "N": world, "causal": w.causal,
                       "l2": "inputs exceed L2 (no flush between steps)",
                       "ring": ring,
                       "parallelism": ("ring over %d real ranks (K/V blocks read in place from the other ranks'"
                                       " memory by the block kernel)" % world) if ring == "peer" else
                                      ("ring over %d real ranks (K/V blocks passed with NCCL point-to-point)"
                                       % world)},
            "pct_bf16_peak": per_gpu / peak_tf,
            "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (block form, one launch per ring step)",
                         "achieved": per_gpu, "peak": peak_tf, "unit": "TFLOP/s", "frac": per_gpu / peak_tf,
                         "peak_source": peak_src + " bf16 burst", "timed": "whole ring per rank, max over ranks",
                         "traffic": None},
            "cpu_baseline": None,
            "e2e": {"value": flops * e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / e_steps},
            "gpu_launches": world * args.steps * (w_launches_dist(world)),
            "clocks": clk,
        }
        emit(line, args)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def w_launches_dist(world):
    """Kernels of this library one rank launches per ring: a block launch per step
    plus, on the last step, the block launch into a partial and the merge that
    writes the output (see ring_dist.ring_attn_fwd_dist)."""
    return world + 1 if world > 1 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.BENCH_WORKLOAD,
                    choices=sorted(n for n, x in W.BY_NAME.items() if x.n_docs == 1))
    ap.add_argument("--mode", default="fused", choices=["fused", "stepwise", "stepwise_epi"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--legs", default="all",
                    help="comma list of merge,configs,backward,allgather,ulysses; 'all' or 'none'")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    ap.add_argument("--jsonl", default=None, help="also append the JSON line to this file")
    ap.add_argument("--ring", default="nccl", choices=["nccl", "peer"],
                    help="with --gpus N > 1: pass the K/V blocks with NCCL (nccl) or read them in place from the"
                         " other ranks' memory (peer)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        return run_dist(args)
    return run_one_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
