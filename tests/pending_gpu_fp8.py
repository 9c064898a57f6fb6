"""FP8 forward parity: attn_fwd_fp8 (through the C ABI) against the fp64
oracle's exact attention of the descaled E4M3 inputs, with the E4M3
tolerances of tests/parity.py.

This module's name keeps it out of pytest's default collection, so that
``pytest tests -m gpu`` does not run it; run it by name on a B200:
``python -m pytest tests/pending_gpu_fp8.py -q``.  Shapes span several
tiles, ragged tails, Nq != Nk and both causal alignments; the long-context
FP8 shape is checked on sampled slices and rows.
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
@pytest.mark.parametrize("nq,nk", [(128, 128), (300, 300), (640, 640), (100, 700), (700, 130), (1, 257)])
def test_fp8_forward_small(causal, nq, nk):
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(2, 2, nq, nk, 128, 3000 + nq + 7 * nk)
    _check(q8, k8, v8, dq, dk, dv, causal, 1 / math.sqrt(128), what=f"fp8 {nq}x{nk} causal={causal}")


def test_fp8_forward_descales_and_scale():
    # Other descale factors and scales: the kernel folds descale_q * descale_k
    # into the scores and descale_v into O.
    q8, k8, v8, _, _, _ = workloads.draw_fp8(1, 2, 384, 384, 128, 3100)
    for dq, dk, dv, scale in ((0.01, 0.02, 0.5, 0.09), (0.003, 0.004, 3.0, 0.2), (0.01, 0.01, 1.0, 0.0)):
        _check(q8, k8, v8, dq, dk, dv, True, scale, what=f"descales {dq} {dk} {dv} scale {scale}")


def test_fp8_forward_constant_v():
    q8, k8, _, dq, dk, _ = workloads.draw_fp8(1, 2, 256, 384, 128, 3200)
    v8 = torch.full((1, 2, 384, 128), 1.0).to(torch.float8_e4m3fn)
    o, _ = _run(q8, k8, v8, dq, dk, 0.75, True, 1 / math.sqrt(128))
    assert torch.all(o.float() == 0.75)


def test_fp8_forward_long_context_sampled():
    w = workloads.FWD_FP8
    n = w["N"]
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(w["B"], w["H"], n, n, w["d"], w["seed"])
    r = np.random.default_rng(n)
    rows = sorted({0, 1, 127, 128, n - 129, n - 128, n - 1, *(int(x) for x in r.choice(n, 40, replace=False))})
    _check(q8, k8, v8, dq, dk, dv, w["causal"], 1 / math.sqrt(w["d"]), slices=[0, 7, w["B"] * w["H"] - 1],
           rows=rows, what="fwd_fp8")


def test_fp8_forward_empty_and_invalid():
    e = torch.empty((1, 1, 0, 128), dtype=torch.float8_e4m3fn, device=DEV)
    k = torch.zeros((1, 1, 128, 128), dtype=torch.float8_e4m3fn, device=DEV)
    o, lse = native.forward_fp8(e, k, k, 1.0, 1.0, 1.0)
    assert o.numel() == 0 and lse.numel() == 0
    with pytest.raises(native.AttnError):
        native.forward_fp8(k[..., :64].contiguous(), k[..., :64].contiguous(), k[..., :64].contiguous(), 1.0, 1.0,
                           1.0)
