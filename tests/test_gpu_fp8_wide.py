"""Wider FP8 forward parity cases: shapes spanning several tiles, ragged
tails, Nq != Nk under each mask, other descale factors and scales, sampled
rows of the long-context FP8 shape, empty or invalid calls, and the packed
variable-length form (attn_fwd_fp8_varlen).
"""

import math

import numpy as np
import pytest
import torch

from exact_attention_150_b200 import native, workloads
from tests.test_gpu_fp8 import DEV, _check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("nq,nk", [(300, 300), (640, 640), (100, 700), (700, 130), (1, 257)])
def test_fp8_forward_small(causal, nq, nk):
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(2, 2, nq, nk, 128, 3000 + nq + 7 * nk)
    _check(q8, k8, v8, dq, dk, dv, causal, 1 / math.sqrt(128), what=f"fp8 {nq}x{nk} causal={causal}")


def test_fp8_forward_descales_and_scale():
    # Other descale factors and scales: the kernel folds descale_q * descale_k
    # into the scores and descale_v into O.
    q8, k8, v8, _, _, _ = workloads.draw_fp8(1, 2, 384, 384, 128, 3100)
    for dq, dk, dv, scale in ((0.01, 0.02, 0.5, 0.09), (0.003, 0.004, 3.0, 0.2), (0.01, 0.01, 1.0, 0.0)):
        _check(q8, k8, v8, dq, dk, dv, True, scale, what=f"descales {dq} {dk} {dv} scale {scale}")


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


@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_fp8_forward_varlen(causal):
    # Packed [H, total, 128] E4M3 batch; each sequence against the oracle on
    # its own rows (empty and one-token sequences included).
    import oracle
    from tests import parity
    lens_q, lens_k = [300, 1, 0, 129, 257], [200, 5, 40, 0, 257]
    H = 2
    tq, tk = sum(lens_q), sum(lens_k)
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(1, H, tq, tk, 128, 3300)
    q8, k8, v8 = (t[0].to(DEV) for t in (q8, k8, v8))
    cu = lambda lens: torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32, device=DEV)
    scale = 1 / math.sqrt(128)
    o, lse = native.forward_fp8_varlen(q8, k8, v8, cu(lens_q), cu(lens_k), max(lens_q), max(lens_k), dq, dk, dv,
                                       causal=causal, scale=scale)
    torch.cuda.synchronize()
    native.device_status()
    o, lse = o.cpu(), lse.cpu()
    qc, kc, vc = (parity.codes(t) for t in (q8, k8, v8))
    a = b = 0
    for nq, nk in zip(lens_q, lens_k):
        oc, off = parity.oracle_mask(causal, nq, nk)
        for h in range(H):
            if nq == 0:
                continue
            if nk == 0:
                assert torch.all(o[h, a:a + nq].float() == 0) and torch.all(torch.isinf(lse[h, a:a + nq]))
                continue
            ref, lref = oracle.forward_fp8(qc[h, a:a + nq], kc[h, b:b + nk], vc[h, b:b + nk], dq, dk, dv, scale, oc,
                                           q_offset=off)
            vmax = float(np.abs(dv * oracle.e4m3_decode(vc[h, b:b + nk])).max())
            parity.assert_o_fp8(parity.f64(o[h, a:a + nq]), ref, vmax, f"seq {nq}x{nk} head {h}")
            parity.assert_lse(parity.f64(lse[h, a:a + nq]), lref, f"seq {nq}x{nk} head {h}")
        a += nq
        b += nk
