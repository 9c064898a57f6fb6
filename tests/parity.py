"""Shared helpers of the GPU parity tests: exact upcasts, per-slice oracle
calls and the tolerance checks.

Tolerances (attention parity bar for this library):
  O:   max |O_gpu - O_ref| <= 2e-3 (fp16) or 1e-2 (bf16);
  LSE: max |LSE_gpu - LSE_ref| <= 1e-3;
  dQ, dK, dV: ||G_gpu - G_ref||_F / ||G_ref||_F <= 2e-2.
FP8 forward (E4M3 inputs, bf16 O), against the oracle's exact attention of
the descaled inputs: the probabilities are rounded to E4M3 (3 mantissa bits)
before the product with V, so O is held to ||dO||_F / ||O_ref||_F <= 5e-2
and max |dO| <= 3e-2 * max |V|, about twice and three times what rounding P
to E4M3 against the exact row maximum gives on N(0, 1) inputs (2.0-2.5e-2
and up to 0.9e-2).  LSE is computed from the unrounded probabilities and
keeps the 1e-3 bar.
O is stored in 16 bits, and half a unit in the last place of a 16-bit
number exceeds the O tolerance once |O| >= 4 (bf16) or >= 8 (fp16): there
not even the correctly rounded exact value meets it.  Those elements are
held to the tolerance plus half a unit in the last place at |O_ref| (a
value within the tolerance before it is rounded to 16 bits is within that
after); every other element is held to the stated tolerance.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

O_TOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}
LSE_TOL = 1e-3
GRAD_TOL = 2e-2
FP8_O_REL_FRO = 5e-2
FP8_O_MAX_ABS_OF_VMAX = 3e-2
_MANT = {torch.float16: 10, torch.bfloat16: 7}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (16-bit or fp32) tensor to a float64 array."""
    return t.detach().to("cpu", torch.float64).numpy()


def ulp16(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return np.exp2(e - _MANT[dtype])


def o_violations(got: np.ndarray, ref: np.ndarray, dtype: torch.dtype) -> tuple[int, float]:
    """Number of O elements outside the bar, and the max abs error."""
    err = np.abs(got - ref)
    half = 0.5 * ulp16(ref, dtype)
    allow = np.where(half > O_TOL[dtype], O_TOL[dtype] + half, O_TOL[dtype])
    return int(np.count_nonzero(err > allow)), float(err.max(initial=0.0))


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_o(got, ref, dtype, what=""):
    n, mx = o_violations(got, ref, dtype)
    assert n == 0, f"{what}: {n} O elements outside tolerance (max abs err {mx:.3e})"


def assert_lse(got, ref, what=""):
    # Rows that see no key have LSE = -inf on both sides; compare the rest.
    inf_got, inf_ref = np.isinf(got), np.isinf(ref)
    assert np.array_equal(inf_got, inf_ref) and np.array_equal(got[inf_ref], ref[inf_ref]), \
        f"{what}: infinite LSE entries differ"
    err = float(np.max(np.abs(got[~inf_ref] - ref[~inf_ref]), initial=0.0))
    assert err <= LSE_TOL, f"{what}: LSE max abs err {err:.3e}"


def assert_grad(got, ref, name, what=""):
    e = rel_fro(got, ref)
    assert e <= GRAD_TOL, f"{what}: {name} relative Frobenius error {e:.3e}"


def oracle_mask(causal, nq: int, nk: int) -> tuple[bool, int]:
    """The oracle's (causal, q_offset) for the library's `causal` argument:
    top-left is offset 0, bottom-right is offset Nk - Nq."""
    if causal in ("bottom_right", 2):
        return True, nk - nq
    if causal in ("none", False, 0):
        return False, 0
    return True, 0


def oracle_forward_slices(q, k, v, scale, causal, slices, rows=None):
    """Oracle O and LSE for the given flat (b*h) slices, optionally only for
    query rows `rows` (absolute indices, ascending)."""
    B, H, Nq, d = q.shape
    causal, off = oracle_mask(causal, Nq, k.shape[2])
    qf, kf, vf = (t.reshape(B * H, t.shape[2], d) for t in (q, k, v))
    outs, lses = [], []
    for s in slices:
        k64, v64 = f64(kf[s]), f64(vf[s])
        if rows is None:
            o, lse, _ = oracle.forward(f64(qf[s]), k64, v64, scale, causal, q_offset=off)
        else:
            o = np.empty((len(rows), d))
            lse = np.empty(len(rows))
            q64 = f64(qf[s])
            for r in rows:  # one row at a time: the oracle sees exactly that query
                oo, ll, _ = oracle.forward(q64[r:r + 1], k64, v64, scale, causal, q_offset=r + off)
                i = rows.index(r)
                o[i], lse[i] = oo[0], ll[0]
        outs.append(o)
        lses.append(lse)
    return outs, lses


def assert_o_fp8(got, ref, v_max_abs, what=""):
    """FP8 forward: O within the E4M3 bars above (v_max_abs = max |V| of the
    descaled values)."""
    e = rel_fro(got, ref)
    assert e <= FP8_O_REL_FRO, f"{what}: O relative Frobenius error {e:.3e}"
    mx = float(np.max(np.abs(got - ref), initial=0.0))
    assert mx <= FP8_O_MAX_ABS_OF_VMAX * v_max_abs, f"{what}: O max abs err {mx:.3e} (max |V| {v_max_abs:.3e})"


def codes(t: torch.Tensor) -> np.ndarray:
    """The byte codes of a torch.float8_e4m3fn tensor, as a numpy array."""
    return t.detach().to("cpu").view(torch.uint8).numpy()
