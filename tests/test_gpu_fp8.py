"""FP8 forward parity: attn_fwd_fp8 (through the C ABI) against the fp64
oracle's exact attention of the descaled E4M3 inputs, with the E4M3
tolerances of tests/parity.py: one 128 x 128 tile per problem under each
mask, and constant V.  tests/test_gpu_fp8_wide.py holds the wider cases.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_150_b200 import native, workloads
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(q8, k8, v8, dq, dk, dv, causal, scale):
    o, lse = native.forward_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), dq, dk, dv, causal=causal, scale=scale)
    torch.cuda.synchronize()
    native.device_status()
    return o.cpu(), lse.cpu()


def _check(q8, k8, v8, dq, dk, dv, causal, scale, slices=None, rows=None, what=""):
    o, lse = _run(q8, k8, v8, dq, dk, dv, causal, scale)
    B, H, Nq, d = q8.shape
    Nk = k8.shape[2]
    oc, off = parity.oracle_mask(causal, Nq, Nk)
    qc, kc, vc = (parity.codes(t).reshape(B * H, -1, d) for t in (q8, k8, v8))
    of, lf = o.reshape(B * H, Nq, d), lse.reshape(B * H, Nq)
    for s in (range(B * H) if slices is None else slices):
        vmax = float(np.abs(dv * oracle.e4m3_decode(vc[s])).max())
        if rows is None:
            ref, lref = oracle.forward_fp8(qc[s], kc[s], vc[s], dq, dk, dv, scale, oc, q_offset=off)
            got_o, got_l = parity.f64(of[s]), parity.f64(lf[s])
        else:
            ref = np.empty((len(rows), d))
            lref = np.empty(len(rows))
            for i, r in enumerate(rows):  # one query row at a time
                oo, ll = oracle.forward_fp8(qc[s][r:r + 1], kc[s], vc[s], dq, dk, dv, scale, oc, q_offset=r + off)
                ref[i], lref[i] = oo[0], ll[0]
            got_o, got_l = parity.f64(of[s][rows]), parity.f64(lf[s][rows])
        parity.assert_o_fp8(got_o, ref, vmax, f"{what} slice {s}")
        parity.assert_lse(got_l, lref, f"{what} slice {s}")


@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_fp8_forward_one_tile(causal):
    nq = nk = 128
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(2, 2, nq, nk, 128, 3000 + nq + 7 * nk)
    _check(q8, k8, v8, dq, dk, dv, causal, 1 / math.sqrt(128), what=f"fp8 {nq}x{nk} causal={causal}")


def test_fp8_forward_constant_v():
    q8, k8, _, dq, dk, _ = workloads.draw_fp8(1, 2, 256, 384, 128, 3200)
    v8 = torch.full((1, 2, 384, 128), 1.0).to(torch.float8_e4m3fn)
    o, _ = _run(q8, k8, v8, dq, dk, 0.75, True, 1 / math.sqrt(128))
    assert torch.all(o.float() == 0.75)
