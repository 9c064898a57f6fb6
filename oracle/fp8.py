"""fp64 CPU oracle for attention over FP8 (E4M3) inputs with per-tensor scales.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
never calls it, and this module imports nothing from the product package.

The page "Flash Attention 是什麼|為何更快又省 VRAM", section "從 FA-1 到 FA-4",
says only that FlashAttention-3 adds an FP8 variant (with lower numerical
error than a baseline FP8 attention); it gives no method.  The reading taken
here is the plainest one: Q, K and V arrive as E4M3 codes q8, k8, v8 with one
fp32 descale factor per tensor, and stand for descale_q * decode(q8) and so
on.  What the FP8 path computes is then exact attention of those real values,
so the oracle is that definition: decode exactly, multiply by the descale
factors, and call the fp64 attention oracle.  The rounding the 8-bit tensor
path adds (the probabilities rounded to E4M3 before the product with V) is
error of the method against this definition, bounded in the tests, not part
of what is computed.

E4M3 here is the OCP 8-bit floating-point format E4M3 ("FN": finite, no
infinities): bit 7 sign, bits 6..3 a biased exponent e (bias 7), bits 2..0 a
mantissa m.  e = 0 encodes the subnormals m * 2^-9; otherwise the value is
(1 + m/8) * 2^(e - 7); e = 15 with m = 7 is NaN (so the largest finite value
is 1.75 * 2^8 = 448).
"""

from __future__ import annotations

import numpy as np

from . import attention

__all__ = ["e4m3_decode", "forward_fp8"]


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes (any integer array with values 0..255) -> float64,
    exactly, from the bit fields of the format."""
    c = np.asarray(codes).astype(np.int64)
    if np.any((c < 0) | (c > 255)):
        raise ValueError("E4M3 codes are bytes")
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = m * 2.0 ** -9
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def forward_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float, scale: float, causal: bool,
                q_offset: int = 0):
    """O, LSE of attention over the real tensors descale_x * decode(x8).

    q8: [..., Nq, d], k8 and v8: [..., Nk, d] byte codes.  Returns the fp64
    attention oracle's O and LSE (natural log of the row sums of
    exp(scale * q_i . k_j) over the unmasked keys, with q and k the
    descaled values).
    """
    q = descale_q * e4m3_decode(q8)
    k = descale_k * e4m3_decode(k8)
    v = descale_v * e4m3_decode(v8)
    o, lse, _ = attention.forward(q, k, v, scale, causal, q_offset)
    return o, lse
