"""The FMA-pipe 2^x of the tensor-core kernel (csrc/exp2_poly.h): the header is what
its generator writes, and the device sequence, emulated step by step in float32,
stays within its relative-error bound against float64 exp2 over the range the
softmax feeds it (scores minus the running max, at most 8 above it)."""
import importlib.util
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GEN = os.path.join(ROOT, "context_attention_cp_b200", "csrc", "gen_exp2_poly.py")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", GEN)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_header_is_current():
    assert subprocess.run([sys.executable, GEN, "--check"]).returncode == 0


def test_relative_error_bound():
    g = _gen()
    coef = g.float32_coefficients()
    assert g.max_relative_error(coef) < 1e-4  # well below bf16 rounding (2^-9)


def test_exact_powers_and_reduction():
    g = _gen()
    coef = g.float32_coefficients()
    xs = np.arange(-120, 9, dtype=np.float32)
    got = g.emulate(xs, coef).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(xs.astype(np.float64)) - 1)) < 1e-4
    # halves land on the reduction boundary f = +-1/2
    hs = np.arange(-40, 8, dtype=np.float32) + np.float32(0.5)
    got = g.emulate(hs, coef).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(hs.astype(np.float64)) - 1)) < 1e-4
