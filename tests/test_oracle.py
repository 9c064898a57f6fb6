"""The fp64 oracle against its pins (no GPU).

Pins: hand-derived closed forms (tests/golden/hand_cases.json), invariants and
special cases of the definition, central finite differences of the backward
pass, the gradient sum identities, a cross-check against an independent
library (torch's fp64 CPU scaled_dot_product_attention and autograd), and
planted mistakes that each must fail at least one pin.
"""

import numpy as np
import pytest
import torch

import oracle
from tests import pins


def test_forward_pins():
    assert pins.forward_pin_failures(oracle.forward) == []


def test_backward_pins():
    assert pins.backward_pin_failures(oracle.backward, oracle.forward) == []


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 5, 5, 3), (2, 3, 17, 17, 8), (1, 1, 64, 64, 16)])
def test_library_crosscheck(causal, shape):
    """torch's fp64 CPU SDPA (top-left causal for square inputs) and autograd."""
    B, H, nq, nk, d = shape
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(B, H, n, d, generator=g, dtype=torch.float64) for n in (nq, nk, nk, nq))
    scale = 0.37
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    o_t = torch.nn.functional.scaled_dot_product_attention(qr, kr, vr, is_causal=causal, scale=scale)
    o_t.backward(do)
    o, lse, _ = oracle.forward(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    np.testing.assert_allclose(o, o_t.detach().numpy(), rtol=1e-12, atol=1e-12)
    s = scale * (q @ k.transpose(-1, -2))
    if causal:
        s = s.masked_fill(torch.ones(nq, nk, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)
    dq, dk, dv = oracle.backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale, causal)
    np.testing.assert_allclose(dq, qr.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kr.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vr.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_query_row_subset_matches_full_problem():
    """Rows [r0, r1) computed alone with q_offset = r0 equal those rows of the
    full problem; this is what the sampled-row parity checks rely on."""
    r = np.random.default_rng(3)
    q, k, v = (r.standard_normal((1, 2, 40, 8)) for _ in range(3))
    for causal in (False, True):
        o, lse, _ = oracle.forward(q, k, v, 0.3, causal)
        o2, lse2, _ = oracle.forward(q[..., 13:29, :], k, v, 0.3, causal, q_offset=13)
        np.testing.assert_allclose(o2, o[..., 13:29, :], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse2, lse[..., 13:29], rtol=1e-13, atol=1e-14)


def test_causal_prefix_and_suffix_windows():
    """Causal: query rows [0, w) depend only on keys [0, w); keys [N-w, N)
    receive gradient only from queries [N-w, N)."""
    r = np.random.default_rng(4)
    n, w = 48, 16
    q, k, v, do = (r.standard_normal((1, 2, n, 8)) for _ in range(4))
    o, lse, _ = oracle.forward(q, k, v, 0.3, True)
    dq, dk, dv = oracle.backward(q, k, v, do, 0.3, True)
    o2, lse2, _ = oracle.forward(q[..., :w, :], k[..., :w, :], v[..., :w, :], 0.3, True)
    np.testing.assert_allclose(o2, o[..., :w, :], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse2, lse[..., :w], rtol=1e-13, atol=1e-14)
    dq2, _, _ = oracle.backward(q[..., :w, :], k[..., :w, :], v[..., :w, :], do[..., :w, :], 0.3, True)
    np.testing.assert_allclose(dq2, dq[..., :w, :], rtol=1e-12, atol=1e-13)
    _, dk3, dv3 = oracle.backward(q[..., n - w:, :], k, v, do[..., n - w:, :], 0.3, True, q_offset=n - w)
    np.testing.assert_allclose(dk3[..., n - w:, :], dk[..., n - w:, :], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv3[..., n - w:, :], dv[..., n - w:, :], rtol=1e-12, atol=1e-13)


# --- planted mistakes: each is the oracle with one plausible error ----------

def _fwd_no_scale(q, k, v, scale, causal, q_offset=0):
    return oracle.forward(q, k, v, 1.0, causal, q_offset)


def _fwd_strict_mask(q, k, v, scale, causal, q_offset=0):
    # masks the diagonal too (j < i instead of j <= i), where a row keeps a key
    if causal:
        o, lse, p = oracle.forward(q, k, v, scale, causal, q_offset - 1)
        return o, lse, p
    return oracle.forward(q, k, v, scale, causal, q_offset)


def _fwd_offset_sign(q, k, v, scale, causal, q_offset=0):
    # diagonal shifted the wrong way (query i sees keys j <= i - offset)
    return oracle.forward(q, k, v, scale, causal, -q_offset)


def _fwd_lse_base2(q, k, v, scale, causal, q_offset=0):
    o, lse, p = oracle.forward(q, k, v, scale, causal, q_offset)
    return o, lse / np.log(2.0), p


def _fwd_reversed_v(q, k, v, scale, causal, q_offset=0):
    o, lse, p = oracle.forward(q, k, v, scale, causal, q_offset)
    return np.matmul(p, np.asarray(v)[..., ::-1, :]), lse, p


def _fwd_column_softmax(q, k, v, scale, causal, q_offset=0):
    s = oracle.scores(q, k, scale, causal, q_offset)
    e = np.exp(s - np.max(s, axis=-2, keepdims=True))
    p = e / e.sum(-2, keepdims=True)
    return np.matmul(p, np.asarray(v, dtype=np.float64)), np.log(np.exp(s).sum(-1)), p


def _fwd_swapped_qk(q, k, v, scale, causal, q_offset=0):
    # S computed as (K Q^T)^T: equal to Q K^T in exact arithmetic, so this
    # rewrite must NOT be flagged
    s = np.swapaxes(oracle.scores(k, q, scale, False), -1, -2)
    if causal:
        nq, nk = s.shape[-2:]
        s = np.where(np.arange(nk)[None, :] > (q_offset + np.arange(nq))[:, None], -np.inf, s)
    # rows that see no key: empty softmax, O = 0, LSE = log 0
    live = np.isfinite(s).any(-1, keepdims=True)
    m = np.where(live, np.max(s, -1, keepdims=True), 0.0)
    e = np.exp(s - m)
    tot = np.where(live, e.sum(-1, keepdims=True), 1.0)
    p = e / tot
    lse = np.where(live, m + np.log(tot), -np.inf)[..., 0]
    return np.matmul(p, np.asarray(v, dtype=np.float64)), lse, p


def _bwd_sign(q, k, v, do, scale, causal, q_offset=0):
    dq, dk, dv = oracle.backward(q, k, v, do, scale, causal, q_offset)
    return -dq, -dk, dv


def _bwd_dk_no_scale(q, k, v, do, scale, causal, q_offset=0):
    dq, dk, dv = oracle.backward(q, k, v, do, scale, causal, q_offset)
    return dq, dk / scale if scale else dk + 1.0, dv


def _bwd_no_d_term(q, k, v, do, scale, causal, q_offset=0):
    _, _, p = oracle.forward(q, k, v, scale, causal, q_offset)
    do = np.asarray(do, dtype=np.float64)
    dv = np.swapaxes(p, -1, -2) @ do
    dp = do @ np.swapaxes(np.asarray(v, dtype=np.float64), -1, -2)
    ds = p * dp                      # forgot "- D"
    return scale * ds @ np.asarray(k, dtype=np.float64), scale * np.swapaxes(ds, -1, -2) @ np.asarray(q, dtype=np.float64), dv


def _bwd_dv_untransposed(q, k, v, do, scale, causal, q_offset=0):
    dq, dk, _ = oracle.backward(q, k, v, do, scale, causal, q_offset)
    _, _, p = oracle.forward(q, k, v, scale, causal, q_offset)
    return dq, dk, p @ np.asarray(do, dtype=np.float64)


@pytest.mark.parametrize("mutant", [_fwd_no_scale, _fwd_strict_mask, _fwd_offset_sign, _fwd_lse_base2,
                                    _fwd_reversed_v, _fwd_column_softmax])
def test_planted_forward_mistakes_are_caught(mutant):
    try:
        fails = pins.forward_pin_failures(mutant)
    except Exception as e:  # a shape error on a pin's input also exposes the mistake
        fails = [repr(e)]
    assert fails, f"{mutant.__name__} passed every pin"


def test_equivalent_rewrite_is_not_flagged():
    """A rewrite that is exact in real arithmetic must pass the pins."""
    assert pins.forward_pin_failures(_fwd_swapped_qk) == []


@pytest.mark.parametrize("mutant", [_bwd_sign, _bwd_dk_no_scale, _bwd_no_d_term, _bwd_dv_untransposed])
def test_planted_backward_mistakes_are_caught(mutant):
    try:
        fails = pins.backward_pin_failures(mutant, oracle.forward)
    except Exception as e:  # a shape error on a pin's input also exposes the mistake
        fails = [repr(e)]
    assert fails, f"{mutant.__name__} passed every pin"
