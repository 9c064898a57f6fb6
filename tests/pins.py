"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics,
checked without retyping the oracle's formula.

Each check takes the forward (and backward) function under test, so that the
same suite can be run against deliberately broken copies of the oracle to show
that a plausible mistake fails at least one pin.

Signatures: fwd(q, k, v, scale, causal, q_offset=0) -> (O, LSE, P) and
bwd(q, k, v, do, scale, causal, q_offset=0) -> (dQ, dK, dV), all float64.
"""

from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _expr(s: str) -> float:
    """Evaluate a golden expression: numbers, + - * / and log()."""
    return float(eval(s, {"__builtins__": {}}, {"log": math.log, "Fraction": Fraction, "inf": math.inf}))


def _mat(rows) -> np.ndarray:
    return np.array([[_expr(x) for x in r] for r in rows], dtype=np.float64)


def golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        return False
    with np.errstate(invalid="ignore"):
        return bool(np.all((a == b) | (np.abs(a - b) <= tol * (1.0 + np.abs(b)))))


def forward_pin_failures(fwd) -> list[str]:
    """Run every forward pin; return the names of those that fail."""
    fails = []
    g = golden_cases()

    # Hand-derived closed forms (golden fixtures).
    for case in g["forward"]:
        q, k, v = _mat(case["q"]), _mat(case["k"]), _mat(case["v"])
        s = _expr(case["scale"])
        # bottom-right: the causal diagonal ends at the last key (offset Nk - Nq).
        for mode, causal, off in (("noncausal", False, 0), ("causal", True, 0),
                                  ("bottom_right", True, k.shape[0] - q.shape[0])):
            if mode not in case:
                continue
            o, lse, _ = fwd(q, k, v, s, causal, off)
            if not _close(o, _mat(case[mode]["o"]), 1e-12):
                fails.append(f"golden {case['name']} {mode} O")
            want_lse = np.array([_expr(x) for x in case[mode]["lse"]])
            if not _close(lse, want_lse, 1e-12):
                fails.append(f"golden {case['name']} {mode} LSE")

    r = _rng(7)
    # Softmax rows sum to one; P is zero where masked; P >= 0.
    for causal in (False, True):
        q, k, v = r.standard_normal((2, 3, 9, 4)), r.standard_normal((2, 3, 11, 4)), r.standard_normal((2, 3, 11, 5))
        _, _, p = fwd(q, k, v, 0.7, causal)
        if np.max(np.abs(p.sum(-1) - 1.0)) > 1e-12 or np.min(p) < 0:
            fails.append(f"rows sum to 1 (causal={causal})")
        if causal and np.any(np.triu(p[..., :9, :9], 1) != 0):
            fails.append("causal P zero above diagonal")
        if causal and np.any(p[..., :, 9:] != 0):
            fails.append("causal P zero for keys past the last query")

    # Constant V returns V's row, for any Q and K.
    for causal in (False, True):
        q, k = r.standard_normal((1, 2, 6, 3)), r.standard_normal((1, 2, 6, 3))
        row = r.standard_normal(4)
        v = np.broadcast_to(row, (1, 2, 6, 4)).copy()
        o, _, _ = fwd(q, k, v, 0.9, causal)
        if not _close(o, np.broadcast_to(row, o.shape), 1e-12):
            fails.append(f"constant V (causal={causal})")

    # First causal query: O_0 = v_0 and LSE_0 = scale * q_0 . k_0.
    q, k, v = r.standard_normal((2, 2, 5, 3)), r.standard_normal((2, 2, 5, 3)), r.standard_normal((2, 2, 5, 3))
    o, lse, _ = fwd(q, k, v, 0.6, True)
    if not _close(o[..., 0, :], v[..., 0, :], 1e-12):
        fails.append("first causal query O")
    if not _close(lse[..., 0], 0.6 * np.sum(q[..., 0, :] * k[..., 0, :], -1), 1e-12):
        fails.append("first causal query LSE")

    # scale = 0: uniform weights; LSE = ln(#visible keys), O = mean of visible V.
    nq = nk = 7
    q, k, v = r.standard_normal((1, 1, nq, 2)), r.standard_normal((1, 1, nk, 2)), r.standard_normal((1, 1, nk, 3))
    o, lse, _ = fwd(q, k, v, 0.0, False)
    if not _close(lse[0, 0], np.full(nq, math.log(nk)), 1e-12) or not _close(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (nq, 3)), 1e-12):
        fails.append("scale 0 non-causal")
    o, lse, _ = fwd(q, k, v, 0.0, True)
    prefix_mean = np.cumsum(v[0, 0], 0) / np.arange(1, nk + 1)[:, None]
    if not _close(lse[0, 0], np.log(np.arange(1, nq + 1)), 1e-12) or not _close(o[0, 0], prefix_mean, 1e-12):
        fails.append("scale 0 causal")

    # A single key: O = v_0.
    q, k, v = r.standard_normal((1, 2, 4, 3)), r.standard_normal((1, 2, 1, 3)), r.standard_normal((1, 2, 1, 3))
    o, lse, _ = fwd(q, k, v, 1.3, False)
    if not _close(o, np.broadcast_to(v, o.shape), 1e-12):
        fails.append("single key")

    # Rows that see no key (causal with a negative offset -m): O = 0,
    # LSE = -inf, P = 0; the other rows are the problem without them.
    m = 3
    q, k, v = r.standard_normal((1, 2, 8, 3)), r.standard_normal((1, 2, 5, 3)), r.standard_normal((1, 2, 5, 4))
    o, lse, p = fwd(q, k, v, 0.8, True, -m)
    if np.any(o[..., :m, :] != 0) or np.any(lse[..., :m] != -np.inf) or np.any(p[..., :m, :] != 0):
        fails.append("rows that see no key")
    o2, lse2, _ = fwd(q[..., m:, :], k, v, 0.8, True, 0)
    if not _close(o[..., m:, :], o2, 1e-12) or not _close(lse[..., m:], lse2, 1e-12):
        fails.append("rows after those that see no key")

    # Permutation equivariance.
    q, k, v = r.standard_normal((2, 3, 8, 4)), r.standard_normal((2, 3, 8, 4)), r.standard_normal((2, 3, 8, 4))
    o, lse, _ = fwd(q, k, v, 0.5, True)
    perm = r.permutation(6)
    sl = lambda x: x.reshape(6, *x.shape[2:])[perm]
    o2, lse2, _ = fwd(sl(q), sl(k), sl(v), 0.5, True)
    if not _close(o2, sl(o), 1e-12) or not _close(lse2, sl(lse), 1e-12):
        fails.append("batch/head permutation")
    o, lse, _ = fwd(q, k, v, 0.5, False)
    pk = r.permutation(8)
    o2, lse2, _ = fwd(q, k[..., pk, :], v[..., pk, :], 0.5, False)
    if not _close(o2, o, 1e-12) or not _close(lse2, lse, 1e-12):
        fails.append("joint key/value row permutation")
    pq = r.permutation(8)
    o2, lse2, _ = fwd(q[..., pq, :], k, v, 0.5, False)
    if not _close(o2, o[..., pq, :], 1e-12) or not _close(lse2, lse[..., pq], 1e-12):
        fails.append("query row permutation")

    # Shift invariance of softmax: adding a constant to every score of a row
    # (k -> k + c*q_dir for the row is awkward; use V shift instead):
    # O(V + c) = O(V) + c because rows of P sum to one.
    c = r.standard_normal(4)
    o3, _, _ = fwd(q, k, v + c, 0.5, False)
    if not _close(o3, o + c, 1e-12):
        fails.append("V shift")
    return fails


def _fd_grads(fwd, q, k, v, do, scale, causal, h=1e-6):
    """Central finite differences of L = sum(O * dO) w.r.t. q, k and v."""
    def loss(qq, kk, vv):
        o, _, _ = fwd(qq, kk, vv, scale, causal)
        return float(np.sum(o * do))
    grads = []
    for which in range(3):
        base = [q, k, v]
        x = base[which]
        gx = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = list(base); args_p[which] = xp
            args_m = list(base); args_m[which] = xm
            gx[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        grads.append(gx)
    return grads


def backward_pin_failures(bwd, fwd) -> list[str]:
    """Run every backward pin; return the names of those that fail.

    ``fwd`` is the trusted forward used for the finite differences.
    """
    fails = []
    g = golden_cases()
    for case in g["backward"]:
        q, k, v, do = (_mat(case[x]) for x in ("q", "k", "v", "do"))
        dq, dk, dv = bwd(q, k, v, do, _expr(case["scale"]), case["causal"], case.get("q_offset", 0))
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            if not _close(got, _mat(case[name]), 1e-12):
                fails.append(f"golden {case['name']} {name}")

    # Central finite differences on tiny inputs (fp64, h = 1e-6).
    r = _rng(11)
    for n, d in ((1, 1), (2, 2), (3, 1), (5, 4), (8, 2)):
        for causal in (False, True):
            q, k, v, do = (r.standard_normal((1, 2, n, d)) for _ in range(4))
            dq, dk, dv = bwd(q, k, v, do, 0.8, causal)
            fq, fk, fv = _fd_grads(fwd, q, k, v, do, 0.8, causal)
            for name, a, b in (("dQ", dq, fq), ("dK", dk, fk), ("dV", dv, fv)):
                err = np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b)))
                if not (err <= 1e-6):
                    fails.append(f"finite differences {name} n={n} d={d} causal={causal}")

    # Rows that see no key add nothing: with offset -m, dQ of the first m
    # rows is 0 and the rest equals the problem without those rows.
    m = 2
    q, do = r.standard_normal((1, 2, 7, 3)), r.standard_normal((1, 2, 7, 4))
    k, v = r.standard_normal((1, 2, 4, 3)), r.standard_normal((1, 2, 4, 4))
    dq, dk, dv = bwd(q, k, v, do, 0.9, True, -m)
    dq2, dk2, dv2 = bwd(q[..., m:, :], k, v, do[..., m:, :], 0.9, True, 0)
    if np.any(dq[..., :m, :] != 0) or not _close(dq[..., m:, :], dq2, 1e-12) or not _close(dk, dk2, 1e-12) \
            or not _close(dv, dv2, 1e-12):
        fails.append("backward rows that see no key")

    # Identities: sum over keys of dK is 0 (rows of dS sum to 0); sum over
    # keys of dV equals sum over queries of dO (columns of P^T sum to 1);
    # scale 0 gives dQ = dK = 0.
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((2, 2, 12, 6)) for _ in range(4))
        dq, dk, dv = bwd(q, k, v, do, 0.4, causal)
        if np.max(np.abs(dk.sum(-2))) > 1e-10:
            fails.append(f"sum of dK over keys (causal={causal})")
        if not _close(dv.sum(-2), do.sum(-2), 1e-10):
            fails.append(f"sum of dV equals sum of dO (causal={causal})")
        dq0, dk0, _ = bwd(q, k, v, do, 0.0, causal)
        if np.max(np.abs(dq0)) > 0 or np.max(np.abs(dk0)) > 0:
            fails.append(f"scale 0 gives zero dQ, dK (causal={causal})")
    return fails
