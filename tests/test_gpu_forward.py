"""Forward parity: the CUDA library (through the C ABI) against the fp64 oracle,
element by element, on seeded inputs.

Small shapes span several tiles, an odd number of query tiles (a CTA with a
single tile) and Nq != Nk.  The named workloads run at full size: every slice
of the tiny, 7B-layer and short sweep workloads, and sampled slices and rows
of the long sweep points and of the long-context workload.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_150_b200 import native, workloads
from exact_attention_150_b200.workloads import draw
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_forward(q, k, v, causal, scale):
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    o, lse = native.forward(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    native.device_status()
    return o.cpu(), lse.cpu()


def check_all_slices(q, k, v, causal, scale, what):
    o, lse = run_forward(q, k, v, causal, scale)
    B, H, Nq, d = q.shape
    refs, lrefs = parity.oracle_forward_slices(q, k, v, scale, causal, range(B * H))
    of, lf = o.reshape(B * H, Nq, d), lse.reshape(B * H, Nq)
    for s in range(B * H):
        parity.assert_o(parity.f64(of[s]), refs[s], q.dtype, f"{what} slice {s}")
        parity.assert_lse(parity.f64(lf[s]), lrefs[s], f"{what} slice {s}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [128, 256, 640])
def test_forward_small(dtype, d, causal, n):
    q, k, v = draw(2, 3, n, n, d, dtype, seed=100 + n + d)
    check_all_slices(q, k, v, causal, 1.0 / math.sqrt(d), f"N{n} d{d} {dtype} causal={causal}")


@pytest.mark.parametrize("nq,nk", [(384, 768), (768, 256), (128, 1024)])
def test_forward_nq_ne_nk(nq, nk):
    q, k, v = draw(1, 2, nq, nk, 128, torch.bfloat16, seed=7)
    check_all_slices(q, k, v, False, 1.0 / math.sqrt(128), f"Nq{nq} Nk{nk}")


@pytest.mark.parametrize("scale", [0.0, -0.3, 0.9])
def test_forward_other_scales(scale):
    q, k, v = draw(1, 2, 256, 256, 64, torch.float16, seed=9)
    for causal in (False, True):
        check_all_slices(q, k, v, causal, scale, f"scale {scale} causal={causal}")


def test_forward_large_scores_need_rescaling():
    """Scores growing along the key axis force the running maximum to move by
    far more than the lazy-rescale threshold on every tile."""
    d = 64
    q, k, v = draw(1, 1, 512, 512, d, torch.bfloat16, seed=11)
    ramp = torch.linspace(0, 6, 512).reshape(1, 1, 512, 1)
    k = (k.float() * 0.2 + ramp).to(torch.bfloat16)
    q = torch.full_like(q, 1.0)
    check_all_slices(q, k, v, False, 1.0, "ramp non-causal")
    check_all_slices(q, k, v, True, 1.0, "ramp causal")


def test_forward_constant_v_and_first_causal_row():
    q, k, v = draw(1, 4, 256, 256, 128, torch.bfloat16, seed=12)
    vc = v[:, :, :1, :].expand_as(v).contiguous()
    o, _ = run_forward(q, k, vc, True, 1 / math.sqrt(128))
    parity.assert_o(parity.f64(o), parity.f64(vc), q.dtype, "constant V")
    o, lse = run_forward(q, k, v, True, 1 / math.sqrt(128))
    assert torch.equal(o[:, :, 0], v[:, :, 0])
    want = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(128)
    np.testing.assert_allclose(lse[:, :, 0].double().numpy(), want.numpy(), atol=1e-4)


def test_forward_unsupported_head_dim_raises():
    q = torch.zeros(1, 1, 128, 96, dtype=torch.float16, device=DEV)
    with pytest.raises(native.AttnError):
        native.forward(q, q, q)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 5, 100, 129, 300, 777])
def test_forward_ragged(dtype, d, causal, n):
    """Lengths that are not multiples of the 128-row tile: the last tile is
    zero-filled by the tensor map, its padding keys are masked and its
    padding query rows are not stored."""
    q, k, v = draw(1, 3, n, n, d, dtype, seed=300 + n + d)
    check_all_slices(q, k, v, causal, 1.0 / math.sqrt(d), f"ragged N{n} d{d} {dtype} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(100, 300), (300, 100), (129, 1), (1, 257), (640, 200)])
def test_forward_ragged_nq_ne_nk(causal, nq, nk):
    """Top-left causal with Nq != Nk: query i sees keys j <= i."""
    q, k, v = draw(2, 2, nq, nk, 128, torch.bfloat16, seed=17 + nq + nk)
    check_all_slices(q, k, v, causal, 1.0 / math.sqrt(128), f"Nq{nq} Nk{nk} causal={causal}")


@pytest.mark.parametrize("nq,nk", [(100, 300), (300, 100), (1, 257), (257, 1), (128, 384), (384, 128),
                                   (640, 200), (200, 640), (129, 129)])
def test_forward_bottom_right(nq, nk):
    """Bottom-right causal: query i sees keys j <= i + Nk - Nq.  With Nq > Nk
    the first Nq - Nk rows see no key: O = 0 and LSE = -inf (whole query
    tiles of such rows are written without any MMA)."""
    q, k, v = draw(2, 2, nq, nk, 128, torch.bfloat16, seed=23 + nq + nk)
    check_all_slices(q, k, v, "bottom_right", 1.0 / math.sqrt(128), f"bottom-right Nq{nq} Nk{nk}")
    if nq > nk:
        o, lse = run_forward(q, k, v, "bottom_right", 0.1)
        assert torch.count_nonzero(o[:, :, :nq - nk]) == 0
        assert torch.all(lse[:, :, :nq - nk] == float("-inf"))
        assert torch.all(torch.isfinite(lse[:, :, nq - nk:]))


@pytest.mark.parametrize("dtype,d", [(torch.float16, 64), (torch.bfloat16, 64), (torch.float16, 128)])
def test_forward_bottom_right_dtypes(dtype, d):
    q, k, v = draw(1, 3, 333, 1000, d, dtype, seed=29)
    check_all_slices(q, k, v, "bottom_right", 1.0 / math.sqrt(d), f"bottom-right d{d} {dtype}")


def test_forward_bottom_right_single_query_is_noncausal():
    """One new query after Nk - 1 cached keys sees all of them."""
    q, k, v = draw(1, 4, 1, 1000, 128, torch.bfloat16, seed=31)
    a = run_forward(q, k, v, "bottom_right", 0.088)
    b = run_forward(q, k, v, False, 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("nq,nk", [(128, 128), (300, 300), (640, 640), (100, 700), (500, 130)])
def test_forward_head_dim_256(dtype, causal, nq, nk):
    """d = 256: Q stays in shared memory, the rounded-P row sums come from
    the softmax threads, and the K/V ring has two slots."""
    q, k, v = draw(1, 2, nq, nk, 256, dtype, seed=41 + nq + nk)
    check_all_slices(q, k, v, causal, 1.0 / math.sqrt(256), f"d256 Nq{nq} Nk{nk} {dtype} causal={causal}")


@pytest.mark.parametrize("scale", [0.0, -0.05])
def test_forward_head_dim_256_other_scales(scale):
    q, k, v = draw(1, 2, 300, 300, 256, torch.bfloat16, seed=47)
    check_all_slices(q, k, v, True, scale, f"d256 scale {scale}")


def test_forward_head_dim_256_varlen():
    lens = [130, 1, 400, 0, 255]
    H, d = 2, 256
    qs, ks, vs = [], [], []
    for b, n in enumerate(lens):
        q, k, v = draw(1, H, n, n, d, torch.bfloat16, seed=51 + b)
        qs.append(q[0]); ks.append(k[0]); vs.append(v[0])
    q, k, v = (torch.cat(t, dim=1).contiguous() for t in (qs, ks, vs))
    cu = torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32)
    o, lse = native.forward_varlen(*(t.to(DEV) for t in (q, k, v)), cu.to(DEV), cu.to(DEV), max(lens), max(lens),
                                   causal=True)
    torch.cuda.synchronize()
    native.device_status()
    o, lse = o.cpu(), lse.cpu()
    for b in range(len(lens)):
        a, z = int(cu[b]), int(cu[b + 1])
        if z == a:
            continue
        for h in range(H):
            ro, rl, _ = oracle.forward(parity.f64(q[h, a:z]), parity.f64(k[h, a:z]), parity.f64(v[h, a:z]),
                                       1 / math.sqrt(d), True)
            parity.assert_o(parity.f64(o[h, a:z]), ro, torch.bfloat16, f"d256 varlen seq {b} head {h}")
            parity.assert_lse(parity.f64(lse[h, a:z]), rl, f"d256 varlen seq {b} head {h}")


def test_forward_empty_problems():
    for shape_q, shape_k in (((0, 2, 128, 64), (0, 2, 128, 64)), ((1, 2, 0, 64), (1, 2, 64, 64))):
        q = torch.zeros(shape_q, dtype=torch.bfloat16, device=DEV)
        k = torch.zeros(shape_k, dtype=torch.bfloat16, device=DEV)
        o, lse = native.forward(q, k, k)
        assert o.numel() == 0 and lse.numel() == 0
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 1, 0, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(native.AttnError):
        native.forward(q, k, k)


# ---------------------------------------------------------- named workloads

def test_tiny_workload():
    w = workloads.TINY
    q, k, v = workloads.make_inputs(w, with_grad=False)
    check_all_slices(q, k, v, w.causal, w.scale, w.label())


def test_layer7b_workload_all_slices():
    w = workloads.LAYER_7B
    q, k, v = workloads.make_inputs(w, with_grad=False)
    check_all_slices(q, k, v, w.causal, w.scale, w.label())


@pytest.mark.parametrize("n", [512, 1024, 2048])
def test_sweep_workload_all_slices(n):
    w = workloads.SWEEP[n]
    q, k, v = workloads.make_inputs(w, with_grad=False)
    check_all_slices(q, k, v, w.causal, w.scale, w.label())


def _sampled_rows(n, count, seed):
    r = np.random.default_rng(seed)
    rows = {0, 1, 127, 128, n - 129, n - 128, n - 1}
    rows.update(int(x) for x in r.choice(n, size=count, replace=False))
    return sorted(x for x in rows if 0 <= x < n)


@pytest.mark.parametrize("n", [4096, 8192])
def test_sweep_workload_sampled(n):
    w = workloads.SWEEP[n]
    q, k, v = workloads.make_inputs(w, with_grad=False)
    o, lse = run_forward(q, k, v, w.causal, w.scale)
    B, H = w.B, w.H
    slices = [0, 37, B * H - 1]
    rows = _sampled_rows(n, 48, n)
    refs, lrefs = parity.oracle_forward_slices(q, k, v, w.scale, w.causal, slices, rows)
    of, lf = o.reshape(B * H, n, w.d), lse.reshape(B * H, n)
    for s, ref, lref in zip(slices, refs, lrefs):
        parity.assert_o(parity.f64(of[s][rows]), ref, q.dtype, f"{w.label()} slice {s}")
        parity.assert_lse(parity.f64(lf[s][rows]), lref, f"{w.label()} slice {s}")


@pytest.mark.parametrize("n", [4096, 8192])
def test_causal_sweep_workload_sampled(n):
    # Causal bf16 on the sweep's batch shape: sampled slices (in different
    # launch groups) and rows, including both sides of tile boundaries.
    w = workloads.CAUSAL_SWEEP[n]
    q, k, v = workloads.make_inputs(w, with_grad=False)
    o, lse = run_forward(q, k, v, w.causal, w.scale)
    B, H = w.B, w.H
    slices = [0, 9, 70, B * H - 1]
    rows = _sampled_rows(n, 48, n + 1)
    refs, lrefs = parity.oracle_forward_slices(q, k, v, w.scale, w.causal, slices, rows)
    of, lf = o.reshape(B * H, n, w.d), lse.reshape(B * H, n)
    for s, ref, lref in zip(slices, refs, lrefs):
        parity.assert_o(parity.f64(of[s][rows]), ref, q.dtype, f"{w.label()} slice {s}")
        parity.assert_lse(parity.f64(lf[s][rows]), lref, f"{w.label()} slice {s}")


@pytest.mark.parametrize("causal", [False, True])
def test_forward_grid_past_the_unit_table(causal):
    """A grid with more work units per CTA than the kernel's set-up table
    holds (256): B64 H32 N2368 d64 is 38,912 query tiles, 263 slots per CTA
    on 148 SMs, so the last units of every CTA are decoded on the fly.
    Those are the last problems of the launch order; slices from the first
    and the last launch group are checked in full against the oracle."""
    B, H, N, d = 64, 32, 2368, 64
    q, k, v = draw(B, H, N, N, d, torch.float16, seed=991 + int(causal))
    o, lse = run_forward(q, k, v, causal, 0.125)
    slices = [0, B * H - 2, B * H - 1]
    refs, lrefs = parity.oracle_forward_slices(q, k, v, 0.125, causal, slices)
    of, lf = o.reshape(B * H, N, d), lse.reshape(B * H, N)
    for s, ref, lref in zip(slices, refs, lrefs):
        parity.assert_o(parity.f64(of[s]), ref, q.dtype, f"unit-table overflow causal={causal} slice {s}")
        parity.assert_lse(parity.f64(lf[s]), lref, f"unit-table overflow causal={causal} slice {s}")
