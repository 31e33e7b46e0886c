"""Shared helpers for the GPU parity tests (inputs from cp_workloads, references
from oracle/, results from the CUDA path through the C ABI)."""
import numpy as np
import torch

# tolerances of the parity bar (max abs error against the fp64 oracle)
TOL = {"bf16": (2e-2, 1e-3), "fp32": (1e-4, 1e-5)}


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close_lse(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), "%s: -inf pattern differs" % what
    assert np.all(got[~fin] == -np.inf), what
    if fin.any():
        err = np.max(np.abs(got[fin] - want[fin]))
        assert err <= tol, "%s: lse max abs err %.3g > %.3g" % (what, err, tol)


def assert_close_o(got, want, tol, what=""):
    err = np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))) if np.size(want) else 0.0
    assert err <= tol, "%s: o max abs err %.3g > %.3g" % (what, err, tol)
    return err


def positions(rng_tuple):
    starts, lens, stride = rng_tuple
    out = []
    for s0, n in zip(starts, lens):
        out.extend(s0 + t * stride for t in range(n))
    return np.array(out, dtype=np.int64)


def sample_rows(w, n_random, seed):
    """(batch, head, original position) triples: position 0, every chunk and rank
    boundary of the layout, plus seeded random ones."""
    from oracle import layout as L
    rng = np.random.default_rng(seed)
    S, N = w.S, w.N
    pos = {0, S - 1}
    c = S // N
    chunk = c // 2 if w.layout == "zigzag" else c
    for p0 in range(0, S, chunk):
        pos.update({p0, min(S - 1, p0 + chunk - 1)})
    for i in range(N):
        rp = L.rank_positions(w.layout, N, S, i) if S <= 1 << 17 else None
        if rp is not None:
            pos.update({rp[0], rp[-1]})
    pos = sorted(pos)
    sel = []
    for k, p in enumerate(pos):
        sel.append((k % w.b, (7 * k) % w.hq, p))
    for _ in range(n_random):
        sel.append((int(rng.integers(w.b)), int(rng.integers(w.hq)), int(rng.integers(S))))
    return np.array(sel, dtype=np.int64)
