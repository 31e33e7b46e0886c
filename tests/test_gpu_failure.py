"""Failure detection on the GPU without faulting it: a kernel's bounded mbarrier wait
is made to run out (nothing ever arrives), the kernel reports through the device
status word and returns, cp_stream_check() turns that into CP_ERR_TIMEOUT and clears
it, and the context keeps working for ordinary calls."""
import numpy as np
import pytest
import torch

import cp_workloads as W
import oracle
from gpu_helpers import TOL, assert_close_lse, assert_close_o, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import context_attention_cp_b200 as m
    m.lib()
    return m


def test_expired_wait_is_reported_and_context_survives(cp):
    torch.cuda.synchronize()
    cp.stream_check()  # start from a clean status word
    cp.selftest_wait_timeout(20_000_000)  # 20 ms
    with pytest.raises(cp.CPError) as err:
        cp.stream_check()
    assert err.value.code == 5  # CP_ERR_TIMEOUT
    cp.stream_check()  # the word was cleared by the first check
    # ordinary work still runs and is right
    q, k, v = W.random_qkv(1, 512, 4, 2, 128, "bf16", seed=77)
    qd, kd, vd = (cp.layout_permute(t.cuda(), "zigzag", 2) for t in (q, k, v))
    o, lse = cp.ring_attn_fwd(qd, kd, vd, "zigzag", 2, True)
    o = cp.layout_permute(o, "zigzag", 2, inverse=True)
    lse = cp.layout_permute(lse, "zigzag", 2, seq_axis=2, inverse=True)
    cp.stream_check()
    ro, rl = oracle.attention(np64(q), np64(k), np64(v), True, 128 ** -0.5)
    assert_close_lse(np64(lse), rl, TOL["bf16"][1])
    assert_close_o(np64(o), ro, TOL["bf16"][0])
