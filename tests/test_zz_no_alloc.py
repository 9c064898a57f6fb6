"""attn_bwd_noalloc: the backward pass for callers that cannot allocate device
memory when they call (a plugin inside another runtime's execution callback,
or a process whose device memory is all held by another allocator's pool).
It uses the library's fixed scratch array instead of a caller workspace.

Checked through the C ABI against attn_bwd (the entry point with a caller
workspace) on two calls in a row with different inputs, so that the second
call runs on scratch that still holds the first call's contents.  This file
is collected last, so a run that stops at its first failure has already run
every other test; it also passes when run alone in a fresh process.
"""

import math

import pytest
import torch

from exact_attention_150_b200 import native
from exact_attention_150_b200.workloads import draw
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
FAKE = 0x10000


def _noalloc(q, k, v, o, lse, do, causal, scale):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    code = native.ATTN_BF16 if q.dtype == torch.bfloat16 else native.ATTN_FP16
    st = native.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Nq, Nk, d,
                                 scale, causal, code, torch.cuda.current_stream().cuda_stream)
    assert st == native.ATTN_OK, native.status_string(st)
    torch.cuda.synchronize()
    native.device_status()
    return dq, dk, dv


@pytest.mark.parametrize("dtype,d,causal", [(torch.bfloat16, 128, True), (torch.float16, 64, False)])
def test_noalloc_matches_attn_bwd_on_two_calls_in_a_row(dtype, d, causal):
    scale = 1.0 / math.sqrt(d)
    for call, seed in enumerate((31, 32)):
        q, k, v, do = (t.to(DEV) for t in draw(2, 4, 1024, 1024, d, dtype, seed=seed, with_grad=True))
        o, lse = native.forward(q, k, v, causal=causal, scale=scale)
        ref = native.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
        got = _noalloc(q, k, v, o, lse, do, causal, scale)
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            parity.assert_grad(parity.f64(g), parity.f64(r), name, f"call {call + 1}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    limit = native.attn_bwd_noalloc_max_scratch_bytes()
    assert limit == 72 << 20
    # 2*16*4096 rows at d=128 need 68 MB: accepted sizes stop just above that.
    assert native.attn_bwd_workspace_bytes(2, 16, 4096, 4096, 128) <= limit
    assert native.attn_bwd_workspace_bytes(4, 16, 4096, 4096, 128) > limit
    st = native.attn_bwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 16, 4096, 4096, 128,
                                 0.1, 1, native.ATTN_BF16, None)
    assert st == native.ATTN_ERR_SCRATCH_LIMIT
    assert "72 MiB" in native.status_string(st)
