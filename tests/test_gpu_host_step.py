"""attn_host_step (host-resident tensors, copies overlapped with the kernels
of other chunks) against the device-resident path on the same inputs.

With the deterministic backward on both sides every output must agree bit
for bit: each chunk runs the same kernels on the same slices.  Cases cover
chunk counts that do not divide B*H, an odd Nq (each chunk's LSE block has
its own alignment), B > 1, both dtypes and the masks.
"""

import math

import pytest
import torch

from exact_attention_150_b200 import native
from exact_attention_150_b200.workloads import draw

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _device_path(q, k, v, do, causal, scale):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = native.forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = native.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale, deterministic=True)
    torch.cuda.synchronize()
    native.device_status()
    return tuple(t.cpu() for t in (o, lse, dq, dk, dv))


@pytest.mark.parametrize("B,H,nq,nk,d,dtype,causal,chunks", [
    (1, 16, 512, 512, 128, torch.bfloat16, True, 4),
    (1, 16, 512, 512, 128, torch.bfloat16, True, 3),      # chunks of 6, 6, 4 slices
    (2, 3, 301, 257, 64, torch.float16, False, 4),        # odd Nq, B > 1, 6 slices in chunks of 2
    (2, 3, 129, 300, 128, torch.float16, "bottom_right", 5),
    (1, 2, 640, 640, 64, torch.bfloat16, True, 1),
    (1, 4, 300, 300, 256, torch.bfloat16, True, 2),       # head dimension 256
])
def test_host_step_matches_device_path(B, H, nq, nk, d, dtype, causal, chunks):
    q, k, v, do = draw(B, H, nq, nk, d, dtype, 4000 + nq + nk, with_grad=True)
    scale = 1 / math.sqrt(d)
    ref = _device_path(q, k, v, do, causal, scale)
    pin = [t.pin_memory() for t in (q, k, v, do)]
    got = native.host_step(*pin, causal=causal, scale=scale, chunks=chunks, deterministic=True, device=DEV)
    torch.cuda.synchronize()
    native.device_status()
    for name, g, r in zip(("o", "lse", "dq", "dk", "dv"), got, ref):
        assert torch.equal(g, r), f"{name} differs from the device path"


def test_host_step_no_queries_zeroes_key_gradients():
    k = torch.randn(1, 2, 128, 64).to(torch.bfloat16)
    q = torch.empty(1, 2, 0, 64, dtype=torch.bfloat16)
    outs = (torch.empty(1, 2, 0, 64, dtype=torch.bfloat16), torch.empty(1, 2, 0),
            torch.empty(1, 2, 0, 64, dtype=torch.bfloat16), torch.full((1, 2, 128, 64), 7.0).to(torch.bfloat16),
            torch.full((1, 2, 128, 64), 7.0).to(torch.bfloat16))
    native.host_step(q, k, k, q, outs=outs, device=DEV)
    torch.cuda.synchronize()
    assert torch.all(outs[3] == 0) and torch.all(outs[4] == 0)
