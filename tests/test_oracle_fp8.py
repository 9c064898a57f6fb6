"""Pins of the FP8 oracle (oracle/fp8.py) against things other than itself:

* the E4M3 decoder against torch's own float8_e4m3fn conversion for all 256
  codes, against values worked by hand from the format's bit fields (OCP
  8-bit floating point specification, E4M3: bias 7, 3 mantissa bits, no
  infinities, S.1111.111 NaN), and for monotonicity;
* the FP8 forward on 2x2 cases worked by hand, on constant V, and on the
  identities the per-tensor scales must satisfy (descale_v scales O only;
  descale_q and descale_k enter only through their product with scale).
"""

import math

import numpy as np
import pytest
import torch

import oracle

# (code, value) worked from the bit fields: sign, e = bits 6..3, m = bits 2..0.
HAND_CODES = [
    (0x00, 0.0),
    (0x01, 2.0 ** -9),            # smallest subnormal: m = 1, e = 0
    (0x07, 7 * 2.0 ** -9),        # largest subnormal
    (0x08, 2.0 ** -6),            # smallest normal: e = 1, m = 0
    (0x38, 1.0),                  # e = 7
    (0x39, 1.125),                # e = 7, m = 1
    (0x40, 2.0),
    (0x48, 4.0),
    (0x50, 8.0),
    (0x77, 1.875 * 2.0 ** 7),     # e = 14, m = 7: 240
    (0x78, 256.0),                # e = 15, m = 0
    (0x7E, 448.0),                # e = 15, m = 6: the largest finite value
    (0xB8, -1.0),
    (0xFE, -448.0),
]


def test_e4m3_decode_hand_values():
    codes = np.array([c for c, _ in HAND_CODES])
    got = oracle.e4m3_decode(codes)
    np.testing.assert_array_equal(got, np.array([v for _, v in HAND_CODES]))
    assert np.signbit(oracle.e4m3_decode(0x80))          # negative zero
    assert np.all(np.isnan(oracle.e4m3_decode([0x7F, 0xFF])))


def test_e4m3_decode_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes.numpy())
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    finite = ~np.isnan(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])


def test_e4m3_decode_is_monotone_and_odd():
    pos = oracle.e4m3_decode(np.arange(0x00, 0x7F))
    assert np.all(np.diff(pos) > 0)
    np.testing.assert_array_equal(oracle.e4m3_decode(np.arange(0x80, 0xFF)), -pos)
    with pytest.raises(ValueError):
        oracle.e4m3_decode([256])


def _hand_problem():
    # d = 1.  q = [1, 0], k = [0, 2], v = [4, 8] as E4M3 codes; with
    # scale = ln(3) / 2, query 0 scores [0, ln 3]: P = [1/4, 3/4], O = 7,
    # LSE = ln 4; query 1 scores [0, 0]: O = 6, LSE = ln 2.
    q8 = np.array([[0x38], [0x00]])
    k8 = np.array([[0x00], [0x40]])
    v8 = np.array([[0x48], [0x50]])
    return q8, k8, v8, math.log(3.0) / 2.0


def test_forward_fp8_hand_case():
    q8, k8, v8, scale = _hand_problem()
    o, lse = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 1.0, scale, causal=False)
    np.testing.assert_allclose(o[:, 0], [7.0, 6.0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, [math.log(4.0), math.log(2.0)], rtol=0, atol=1e-12)
    # Causal: query 0 sees only key 0 (O = 4, LSE = 0); query 1 is unchanged.
    o, lse = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 1.0, scale, causal=True)
    np.testing.assert_allclose(o[:, 0], [4.0, 6.0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, [0.0, math.log(2.0)], rtol=0, atol=1e-12)


def test_forward_fp8_hand_case_with_descales():
    # descale_q = 2 and scale halved give the same scores; descale_v = 0.5
    # halves O and leaves LSE alone.
    q8, k8, v8, scale = _hand_problem()
    o, lse = oracle.forward_fp8(q8, k8, v8, 2.0, 1.0, 0.5, scale / 2.0, causal=False)
    np.testing.assert_allclose(o[:, 0], [3.5, 3.0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, [math.log(4.0), math.log(2.0)], rtol=0, atol=1e-12)


def _random_codes(rng, shape):
    # Finite codes only (0x7F and 0xFF are NaN), with a magnitude cap so the
    # scores stay moderate.
    c = rng.integers(0, 0x60, size=shape)
    return np.where(rng.random(shape) < 0.5, c, c | 0x80)


@pytest.mark.parametrize("causal", [False, True])
def test_forward_fp8_scale_identities(causal):
    rng = np.random.default_rng(5)
    q8, k8, v8 = (_random_codes(rng, (2, 9, 8)), _random_codes(rng, (2, 11, 8)), _random_codes(rng, (2, 11, 8)))
    base_o, base_l = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 1.0, 0.01, causal)
    # descale_v enters O linearly and nothing else.
    o, lse = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 3.0, 0.01, causal)
    np.testing.assert_allclose(o, 3.0 * base_o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, base_l, rtol=1e-13, atol=1e-13)
    # descale_q and descale_k act only through scale * descale_q * descale_k.
    o1, l1 = oracle.forward_fp8(q8, k8, v8, 0.5, 4.0, 1.0, 0.01, causal)
    o2, l2 = oracle.forward_fp8(q8, k8, v8, 4.0, 0.5, 1.0, 0.01, causal)
    o3, l3 = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 1.0, 0.02, causal)
    for o_, l_ in ((o2, l2), (o3, l3)):
        np.testing.assert_allclose(o_, o1, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(l_, l1, rtol=1e-12, atol=1e-12)
    assert not np.allclose(o1, base_o)  # the scores did change


def test_forward_fp8_constant_v():
    rng = np.random.default_rng(6)
    q8, k8 = _random_codes(rng, (3, 5, 4)), _random_codes(rng, (3, 7, 4))
    v8 = np.full((3, 7, 4), 0x38)  # every value 1.0
    o, _ = oracle.forward_fp8(q8, k8, v8, 1.0, 1.0, 0.25, 0.3, causal=True)
    np.testing.assert_allclose(o, 0.25, rtol=0, atol=1e-14)


def _emulated_fp8_forward(q8, k8, v8, dq, dk, dv, scale, causal, drop_v_descale=False, drop_qk_descale=False):
    # The 8-bit path's arithmetic on the CPU: P = exp(S - row max) rounded to
    # E4M3 by torch's conversion, O = (P V) / (sum of the rounded P), bf16.
    q = oracle.e4m3_decode(q8) * (1.0 if drop_qk_descale else dq)
    k = oracle.e4m3_decode(k8) * (1.0 if drop_qk_descale else dk)
    v = oracle.e4m3_decode(v8) * (1.0 if drop_v_descale else dv)
    s = oracle.scores(q, k, scale, causal)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    pr = torch.from_numpy(p.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    o = (pr @ v) / pr.sum(axis=-1, keepdims=True)
    return torch.from_numpy(o).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("n,causal", [(128, False), (384, True), (700, False)])
def test_fp8_tolerance_admits_e4m3_rounding_and_rejects_mistakes(n, causal):
    from exact_attention_150_b200 import workloads
    from tests import parity
    q8t, k8t, v8t, dq, dk, dv = workloads.draw_fp8(1, 2, n, n, 128, 2000 + n)
    scale = 1 / math.sqrt(128)
    for s in range(2):
        q8, k8, v8 = (parity.codes(t)[0, s] for t in (q8t, k8t, v8t))
        ref, _ = oracle.forward_fp8(q8, k8, v8, dq, dk, dv, scale, causal)
        vmax = float(np.abs(dv * oracle.e4m3_decode(v8)).max())
        parity.assert_o_fp8(_emulated_fp8_forward(q8, k8, v8, dq, dk, dv, scale, causal), ref, vmax)
        for mistake in ("drop_v_descale", "drop_qk_descale"):
            bad = _emulated_fp8_forward(q8, k8, v8, dq, dk, dv, scale, causal, **{mistake: True})
            with pytest.raises(AssertionError):
                parity.assert_o_fp8(bad, ref, vmax)
        # V's key rows in the wrong order (a mis-addressed operand) is caught.
        bad = _emulated_fp8_forward(q8, k8, v8[::-1].copy(), dq, dk, dv, scale, causal)
        with pytest.raises(AssertionError):
            parity.assert_o_fp8(bad, ref, vmax)
