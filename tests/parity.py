"""Comparison helpers shared by the GPU parity tests, smoke() and bench.py's checks.

Tolerances (from the stated targets of the hot path):
  - slot indices: bit-exact, except where the oracle's score gap at the W / R boundary
    is below 1e-5 (near ties, counted and reported, never failed);
  - outputs and final memory: normwise max relative error per (b,h) tensor,
    max|x - y| / max|y|, at most 1e-4 for fp32 inputs and 2e-2 for bf16 inputs
    (fp32 state in both cases).
"""
from __future__ import annotations

import os

import numpy as np

SCORE_GAP = 1e-5
TOL = {"f32": 1e-4, "bf16": 2e-2}


def normwise_rel_err(x, y) -> float:
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.abs(y).max()
    if den == 0:
        return float(np.abs(x).max())
    return float(np.abs(x - y).max() / den)


def per_bh_rel_err(x, y) -> float:
    """Largest normwise relative error over the leading (b,h) axes of [B,H,...] arrays."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    B, H = x.shape[:2]
    return max(normwise_rel_err(x[b, h], y[b, h]) for b in range(B) for h in range(H))


def slot_scores(orc, x_vec, sk_head, slots, n):
    """Oracle (fp64) scores of arbitrary slots for one vector."""
    s1, s2 = orc.half_scores(x_vec, sk_head)
    slots = np.asarray(slots)
    return s1[slots // n] + s2[slots % n]


def compare_selection(orc, x, sk, gpu_idx, ora_idx, ora_score, n, gap=SCORE_GAP):
    """Compare GPU and oracle top-k selections row by row.

    x [B,H,T,d_k] (the rows scored), sk [H,2,n,h], *_idx [B,H,T,top], ora_score the
    oracle's sorted scores.  Returns (exact_rows, near_tie_rows, bad_rows, details).
    A row is a near tie when the two selections differ only by slots whose oracle
    scores lie within `gap` of the oracle's boundary score, and the GPU's order agrees
    with the oracle scores up to `gap`.
    """
    gpu_idx = np.asarray(gpu_idx)
    ora_idx = np.asarray(ora_idx)
    B, H, T, top = gpu_idx.shape
    exact = near = 0
    bad = []
    rows = np.argwhere(np.any(gpu_idx != ora_idx, axis=-1))
    exact = B * H * T - len(rows)
    for (b, h, t) in rows:
        g = gpu_idx[b, h, t]
        o = ora_idx[b, h, t]
        thr = ora_score[b, h, t, -1]
        gs = slot_scores(orc, x[b, h, t], sk[h], g, n)
        ok = True
        if len(set(g.tolist())) != top or np.any(g < 0) or np.any(g >= n * n):
            ok = False
        only_g = [s for s in g.tolist() if s not in set(o.tolist())]
        only_o = [s for s in o.tolist() if s not in set(g.tolist())]
        if only_g:
            sg = slot_scores(orc, x[b, h, t], sk[h], only_g, n)
            ok &= bool(np.all(sg >= thr - gap))
        if only_o:
            so = slot_scores(orc, x[b, h, t], sk[h], only_o, n)
            ok &= bool(np.all(so <= thr + gap))
        ok &= bool(np.all(np.diff(gs) <= gap))  # GPU order follows the scores
        if ok:
            near += 1
        else:
            bad.append((int(b), int(h), int(t)))
    return exact, near, bad


def f64(t):
    """torch tensor (any device / dtype) -> fp64 numpy."""
    return t.detach().to("cpu").double().numpy()


# Observed errors of every tolerance check in this process, (test id, what, error, tolerance),
# printed by the terminal summary so that drift well inside a tolerance stays visible.
OBSERVED: list[tuple[str, str, float, float]] = []


def check_err(err: float, tol: float, what: str = "rel err") -> float:
    """Record an observed error and fail, naming it, when it exceeds its tolerance."""
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    OBSERVED.append((test, what, float(err), float(tol)))
    assert err <= tol, f"{what}: max rel err {err:.3e} above tolerance {tol:.1e}"
    return err
