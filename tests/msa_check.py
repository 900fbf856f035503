"""Comparison rules shared by the parity tests (selection sets with near-ties, error metrics).

The selection rule: a GPU block set is accepted for a query iff it equals the oracle's set
except for blocks whose fp64 score lies within ``REL_TIE`` (relative) of the oracle's 15th
best score; each such block is a logged near-tie. When the 15th score is itself close to
zero, the relative window is measured against the sum of |q_i * kbar_i| / sqrt(d_I) of the
block instead (a "cancellation near-tie", counted separately).
"""
from __future__ import annotations

import numpy as np

REL_TIE = 1e-5
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


def compare_selection_row(gpu_sel, ora_sel, scores, kth, abs_scale=None):
    """Returns (ok, n_near_tie, n_cancel_tie). gpu_sel/ora_sel: int arrays (-1 padded);
    scores: fp64 oracle scores of all candidates (index = block id); kth: oracle 15th score;
    abs_scale: per-candidate sum |q_i kbar_i| / sqrt(dI) (optional)."""
    g = set(int(v) for v in gpu_sel if v >= 0)
    o = set(int(v) for v in ora_sel if v >= 0)
    if len(g) != len([v for v in gpu_sel if v >= 0]):
        return False, 0, 0          # duplicates
    if len(g) != len(o):
        return False, 0, 0
    diff = g ^ o
    if not diff:
        return True, 0, 0
    if np.isnan(kth):
        return False, 0, 0
    near = cancel = 0
    for b in diff:
        if b >= len(scores):
            return False, 0, 0      # diagonal or out of range: must match exactly
        dlt = abs(scores[b] - kth)
        if dlt <= REL_TIE * abs(kth):
            near += 1
        elif abs_scale is not None and dlt <= REL_TIE * abs_scale[b]:
            cancel += 1
        else:
            return False, near, cancel
    return True, near, cancel


def sel_sorted_ok(sel_row) -> bool:
    """Valid ids ascending, then only -1 padding."""
    s = list(sel_row)
    n = sum(1 for v in s if v >= 0)
    valid = s[:n]
    return all(v < 0 for v in s[n:]) and all(valid[i] < valid[i + 1] for i in range(n - 1))


def error_metrics(gpu: np.ndarray, ref: np.ndarray):
    e = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


def assert_close_attention(gpu, ref, what=""):
    mx, mn = error_metrics(gpu, ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS_TOL, f"{what}: max abs err {mx:.3e} > {MAX_ABS_TOL}"
    assert mn <= MEAN_ABS_TOL, f"{what}: mean abs err {mn:.3e} > {MEAN_ABS_TOL}"
    return mx, mn
