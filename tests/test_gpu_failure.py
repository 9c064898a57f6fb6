"""Failure detection on the GPU without a fault: a bounded wait that runs out
reports ATTN_ERR_TIMEOUT through the device status word, the other role of
the CTA leaves through the abort flag, and the context stays usable."""

import math

import pytest
import torch

import oracle
from exact_attention_150_b200 import native
from exact_attention_150_b200.workloads import draw
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_wait_on_a_barrier_nothing_sets_times_out_and_is_reported():
    torch.cuda.synchronize()
    assert native.attn_last_device_status() == native.ATTN_OK  # nothing pending from earlier tests
    result = torch.full((2,), 7, dtype=torch.int32, device=DEV)
    assert native.selftest_wait_timeout(20000, result) == native.ATTN_OK  # 20 ms limit
    assert native.attn_last_device_status() == native.ATTN_ERR_TIMEOUT
    assert result.cpu().tolist() == [0, 0]  # the timed-out warp and the one that left on the abort flag
    assert native.attn_last_device_status() == native.ATTN_OK  # reading clears the word
    with pytest.raises(native.AttnError, match="status 4"):
        native.selftest_wait_timeout(1000, result)
        native.device_status()


def test_context_is_usable_after_a_timeout():
    result = torch.zeros(2, dtype=torch.int32, device=DEV)
    native.selftest_wait_timeout(5000, result)
    assert native.attn_last_device_status() == native.ATTN_ERR_TIMEOUT
    q, k, v = draw(1, 2, 300, 300, 64, torch.bfloat16, seed=901)
    o, lse = native.forward(*(t.to(DEV) for t in (q, k, v)), causal=True)
    torch.cuda.synchronize()
    native.device_status()
    for s in range(2):
        ro, rl, _ = oracle.forward(parity.f64(q[0, s]), parity.f64(k[0, s]), parity.f64(v[0, s]), 1 / math.sqrt(64), True)
        parity.assert_o(parity.f64(o[0, s].cpu()), ro, torch.bfloat16, "after timeout")
        parity.assert_lse(parity.f64(lse[0, s].cpu()), rl, "after timeout")
