"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product package.

What it computes is the plain three-step definition of attention stated on the
page "FlashAttention 核心原理" (cxbdf.cn), part 1, formula
``Attention(Q, K, V) = softmax((Q * K^T) / sqrt(d_k)) * V`` and the three steps
listed under it (score matrix S = QK^T, row softmax, aggregation with V).  The
score matrix is materialised in full; nothing is tiled, fused or reordered.
FlashAttention's tiled online softmax reaches this same result up to floating
point reordering (same page, part 3, "precise computation"; page "Flash
Attention 是什麼", section "exact, not an approximation"), so this definition is
the oracle.

Readings of the pages taken here (the pages leave these open):

* the scale is a caller argument; the pages' formula uses 1/sqrt(d_k);
* causal masking is top-left aligned: query i sees key j iff j <= i + q_offset,
  where q_offset is the absolute index of the first query row passed in
  (0 for a full problem).  Masked scores are excluded from the softmax;
* LSE is the natural log of sum_j exp(scale * q_i . k_j) over unmasked j, one
  float per query row (the "float* softmax_lse" output in the kernel interface
  sketched on page "FlashAttention-2 性能革命", section 2.1);
* the backward pass is the derivative of the same definition (the pages only
  say that it recomputes the attention matrix instead of storing it: page
  "FlashAttention 核心原理", part 2 item 3).  With P = softmax(S):
  dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij, dS = P * (dP - D),
  dQ = scale * dS K, dK = scale * dS^T Q.

Every array is float64.  Leading dimensions (batch, heads) broadcast.
"""

from __future__ import annotations

import numpy as np

__all__ = ["scores", "forward", "backward"]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def scores(q, k, scale: float, causal: bool, q_offset: int = 0) -> np.ndarray:
    """Step 1 of the definition: S = scale * Q K^T, with -inf where masked.

    q: [..., Nq, d], k: [..., Nk, d].  Returns S: [..., Nq, Nk].
    """
    q = _f64(q)
    k = _f64(k)
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    if causal:
        nq, nk = s.shape[-2], s.shape[-1]
        qpos = q_offset + np.arange(nq)[:, None]
        kpos = np.arange(nk)[None, :]
        s = np.where(kpos > qpos, -np.inf, s)
    return s


def forward(q, k, v, scale: float, causal: bool, q_offset: int = 0):
    """Steps 1-3 of the definition.

    Returns (O [..., Nq, dv], LSE [..., Nq], P [..., Nq, Nk]).
    Rows with every key masked (possible only when q_offset < 0) get O = 0 and
    LSE = -inf.
    """
    v = _f64(v)
    s = scores(q, k, scale, causal, q_offset)
    # Step 2: row softmax.  Subtracting the row maximum only avoids overflow;
    # it cancels in the ratio below.
    m = np.max(s, axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    row_sum = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(row_sum > 0, e / row_sum, 0.0)
        lse = np.where(row_sum[..., 0] > 0, m_safe[..., 0] + np.log(row_sum[..., 0]), -np.inf)
    # Step 3: aggregate V with the probabilities.
    o = np.matmul(p, v)
    return o, lse, p


def backward(q, k, v, do, scale: float, causal: bool, q_offset: int = 0):
    """Gradients of L = sum(O * dO) with respect to Q, K and V.

    dQ has one row per query row passed in.  dK and dV are the contributions of
    the query rows passed in; they are the full gradients when every query row
    of the problem is passed (q_offset = 0, all rows).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    _, _, p = forward(q, k, v, scale, causal, q_offset)
    dv = np.matmul(np.swapaxes(p, -1, -2), do)
    dp = np.matmul(do, np.swapaxes(v, -1, -2))
    d_row = np.sum(p * dp, axis=-1, keepdims=True)
    ds = p * (dp - d_row)
    dq = scale * np.matmul(ds, k)
    dk = scale * np.matmul(np.swapaxes(ds, -1, -2), q)
    return dq, dk, dv
