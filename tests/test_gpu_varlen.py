"""Packed variable-length batches (attn_fwd_varlen / attn_bwd_varlen) against
the fp64 oracle, sequence by sequence, and against the dense calls.

Each sequence is an attention problem of its own: the oracle is run on its
rows alone.  Sequences of equal length packed together must give exactly
the dense result (the kernels do the same tile arithmetic)."""

import math

import pytest
import torch

import oracle
from exact_attention_150_b200 import native
from exact_attention_150_b200.workloads import draw
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def pack(lens_q, lens_k, H, d, dtype, seed):
    """Per-sequence seeded tensors, packed head-major: [H, total, d]."""
    qs, ks, vs, dos = [], [], [], []
    for b, (nq, nk) in enumerate(zip(lens_q, lens_k)):
        q, k, v, do = draw(1, H, max(nq, nk), max(nq, nk), d, dtype, seed=seed + b, with_grad=True)
        qs.append(q[0, :, :nq]); dos.append(do[0, :, :nq]); ks.append(k[0, :, :nk]); vs.append(v[0, :, :nk])
    cat = lambda ts: torch.cat(ts, dim=1).contiguous()
    cu = lambda lens: torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    return cat(qs), cat(ks), cat(vs), cat(dos), cu(lens_q), cu(lens_k)


def run(lens_q, lens_k, H, d, dtype, causal, seed, deterministic=False):
    q, k, v, do, cuq, cuk = pack(lens_q, lens_k, H, d, dtype, seed)
    dev = [t.to(DEV) for t in (q, k, v, do, cuq, cuk)]
    mq, mk = max(lens_q), max(lens_k)
    scale = 1.0 / math.sqrt(d)
    o, lse = native.forward_varlen(dev[0], dev[1], dev[2], dev[4], dev[5], mq, mk, causal=causal, scale=scale)
    dq, dk, dv = native.backward_varlen(dev[0], dev[1], dev[2], o, lse, dev[3], dev[4], dev[5], mq, mk,
                                        causal=causal, scale=scale, deterministic=deterministic)
    torch.cuda.synchronize()
    native.device_status()
    return (q, k, v, do, cuq, cuk), tuple(t.cpu() for t in (o, lse, dq, dk, dv))


def check_against_oracle(inputs, outputs, causal, d, dtype, tag):
    q, k, v, do, cuq, cuk = inputs
    o, lse, dq, dk, dv = outputs
    H = q.shape[0]
    scale = 1.0 / math.sqrt(d)
    for b in range(len(cuq) - 1):
        q0, q1, k0, k1 = int(cuq[b]), int(cuq[b + 1]), int(cuk[b]), int(cuk[b + 1])
        for h in range(H):
            what = f"{tag} seq {b} ({q1 - q0}x{k1 - k0}) head {h}"
            if q1 == q0:
                if k1 > k0:  # no queries: no gradient reaches these keys
                    assert torch.count_nonzero(dk[h, k0:k1]) == 0 and torch.count_nonzero(dv[h, k0:k1]) == 0, what
                continue
            if k1 == k0:  # no keys: empty softmax
                assert torch.count_nonzero(o[h, q0:q1]) == 0, what
                assert torch.all(lse[h, q0:q1] == float("-inf")), what
                assert torch.count_nonzero(dq[h, q0:q1]) == 0, what
                continue
            args = [parity.f64(t[h, a:z]) for t, a, z in ((q, q0, q1), (k, k0, k1), (v, k0, k1), (do, q0, q1))]
            oc, off = parity.oracle_mask(causal, q1 - q0, k1 - k0)
            ro, rl, _ = oracle.forward(*args[:3], scale, oc, off)
            rdq, rdk, rdv = oracle.backward(*args, scale, oc, off)
            parity.assert_o(parity.f64(o[h, q0:q1]), ro, dtype, what)
            parity.assert_lse(parity.f64(lse[h, q0:q1]), rl, what)
            parity.assert_grad(parity.f64(dq[h, q0:q1]), rdq, "dQ", what)
            parity.assert_grad(parity.f64(dk[h, k0:k1]), rdk, "dK", what)
            parity.assert_grad(parity.f64(dv[h, k0:k1]), rdv, "dV", what)


@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float16, 64), (torch.bfloat16, 256),
                                     (torch.float16, 256)])
def test_varlen_self_attention(causal, dtype, d):
    lens = [1, 130, 0, 257, 64, 500]
    inputs, outputs = run(lens, lens, 2, d, dtype, causal, seed=801)
    check_against_oracle(inputs, outputs, causal, d, dtype, f"varlen self {dtype} d{d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("d", [64, 256])
def test_varlen_cross_lengths(causal, d):
    """Different query and key lengths per sequence, including a sequence
    with queries and no keys and one with keys and no queries."""
    lens_q = [100, 3, 300, 0, 50]
    lens_k = [200, 50, 1, 70, 0]
    inputs, outputs = run(lens_q, lens_k, 3, d, torch.bfloat16, causal, seed=811)
    check_against_oracle(inputs, outputs, causal, d, torch.bfloat16, f"varlen cross d{d} causal={causal}")


@pytest.mark.parametrize("d", [128, 256])
def test_varlen_equal_lengths_match_dense_bitwise(d):
    B, H, N = 3, 2, 384
    q, k, v, do = draw(B, H, N, N, d, torch.bfloat16, seed=821, with_grad=True)
    dev = [t.to(DEV) for t in (q, k, v, do)]
    o, lse = native.forward(*dev[:3], causal=True)
    dq, dk, dv = native.backward(*dev[:3], o, lse, dev[3], causal=True)
    packed = [t.permute(1, 0, 2, 3).reshape(H, B * N, d).contiguous() for t in dev]
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device=DEV)
    o2, lse2 = native.forward_varlen(*packed[:3], cu, cu, N, N, causal=True)
    dq2, dk2, dv2 = native.backward_varlen(*packed[:3], o2, lse2, packed[3], cu, cu, N, N, causal=True,
                                           deterministic=True)
    dq3, _, _ = native.backward(*dev[:3], o, lse, dev[3], causal=True, deterministic=True)
    torch.cuda.synchronize()
    native.device_status()
    unpack = lambda t: t.reshape(H, B, N, -1).permute(1, 0, 2, 3)
    assert torch.equal(unpack(o2), o)
    assert torch.equal(lse2.reshape(H, B, N).permute(1, 0, 2), lse)
    assert torch.equal(unpack(dk2), dk) and torch.equal(unpack(dv2), dv)
    assert torch.equal(unpack(dq2), dq3)  # both ordered: identical bits


def test_varlen_deterministic_is_reproducible():
    lens = [700, 1200, 33, 900]
    a = run(lens, lens, 4, 128, torch.bfloat16, True, seed=831, deterministic=True)[1]
    b = run(lens, lens, 4, 128, torch.bfloat16, True, seed=831, deterministic=True)[1]
    for x, y in zip(a, b):
        assert torch.equal(x, y)
