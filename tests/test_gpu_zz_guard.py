"""Out-of-bounds writes: every output and the workspace sit between guard
bands (tests/guard.py), and after the forward and the backward the bands
must be untouched and the results bit-identical to an unguarded run (the
deterministic backward, so dQ is reproducible).  Shapes have ragged query
and key tails, rows that see no key, and a packed variable-length batch, the
places where a stray store would land just past a tensor's end."""

import math

import pytest
import torch

from exact_attention_150_b200 import native
from exact_attention_150_b200.workloads import draw
from tests import guard

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(q, k, v, do, causal, scale, outs=None, ws=None):
    o, lse, dq, dk, dv = outs if outs is not None else (None,) * 5
    o, lse = native.forward(q, k, v, causal=causal, scale=scale, out=o, lse=lse)
    dq, dk, dv = native.backward(q, k, v, o, lse, do, causal=causal, scale=scale, dq=dq, dk=dk, dv=dv,
                                 workspace=ws, deterministic=True)
    torch.cuda.synchronize()
    native.device_status()
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("B,H,nq,nk,d,dtype,causal", [
    (2, 3, 300, 257, 128, torch.bfloat16, True),
    (1, 2, 129, 1, 64, torch.float16, False),
    (2, 2, 1, 300, 128, torch.float16, True),
    (1, 3, 640, 200, 64, torch.bfloat16, "bottom_right"),   # rows that see no key
    (1, 2, 200, 640, 128, torch.bfloat16, "bottom_right"),
])
def test_dense_outputs_stay_inside_their_buffers(B, H, nq, nk, d, dtype, causal):
    q, k, v, do = (t.to(DEV) for t in draw(B, H, nq, nk, d, dtype, 5000 + nq + nk, with_grad=True))
    scale = 1 / math.sqrt(d)
    ref = _run(q, k, v, do, causal, scale)
    shapes = [((B, H, nq, d), dtype), ((B, H, nq), torch.float32), ((B, H, nq, d), dtype), ((B, H, nk, d), dtype),
              ((B, H, nk, d), dtype)]
    held = [guard.guarded(s, t, DEV) for s, t in shapes]
    ws, ws_buf = guard.guarded((native.attn_bwd_workspace_bytes(B, H, nq, nk, d),), torch.uint8, DEV)
    got = _run(q, k, v, do, causal, scale, outs=[t for t, _ in held], ws=ws)
    for name, (_, buf) in zip(("o", "lse", "dq", "dk", "dv"), held):
        assert guard.intact(buf), f"a kernel wrote outside {name}"
    assert guard.intact(ws_buf), "a kernel wrote outside the workspace"
    for name, g, r in zip(("o", "lse", "dq", "dk", "dv"), got, ref):
        assert torch.equal(g, r), f"{name} differs from the unguarded run"


def test_packed_outputs_stay_inside_their_buffers():
    H, d, dtype = 2, 128, torch.bfloat16
    lens = [300, 1, 129, 0, 257]
    total = sum(lens)
    cu = torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32, device=DEV)
    q, k, v, do = (t[0].to(DEV) for t in draw(1, H, total, total, d, dtype, 5100, with_grad=True))
    mx = max(lens)
    scale = 1 / math.sqrt(d)

    def run(outs=None, ws=None):
        o, lse, dq, dk, dv = outs if outs is not None else (None,) * 5
        o, lse = native.forward_varlen(q, k, v, cu, cu, mx, mx, causal=True, scale=scale, out=o, lse=lse)
        dq, dk, dv = native.backward_varlen(q, k, v, o, lse, do, cu, cu, mx, mx, causal=True, scale=scale, dq=dq,
                                            dk=dk, dv=dv, workspace=ws, deterministic=True)
        torch.cuda.synchronize()
        native.device_status()
        return o, lse, dq, dk, dv

    ref = run()
    shapes = [((H, total, d), dtype), ((H, total), torch.float32), ((H, total, d), dtype), ((H, total, d), dtype),
              ((H, total, d), dtype)]
    held = [guard.guarded(s, t, DEV) for s, t in shapes]
    ws, ws_buf = guard.guarded((native.attn_bwd_varlen_workspace_bytes(len(lens), H, total, mx, d),), torch.uint8,
                               DEV)
    got = run(outs=[t for t, _ in held], ws=ws)
    for name, (_, buf) in zip(("o", "lse", "dq", "dk", "dv"), held):
        assert guard.intact(buf), f"a kernel wrote outside {name}"
    assert guard.intact(ws_buf), "a kernel wrote outside the workspace"
    for name, g, r in zip(("o", "lse", "dq", "dk", "dv"), got, ref):
        assert torch.equal(g, r), f"{name} differs from the unguarded run"
