"""Comparison rules shared by the parity tests (selection sets with near-ties, error metrics).

Selection rule. A GPU block set is accepted for a query iff it equals the oracle's set except
for blocks whose fp64 score lies within ``REL_TIE`` (relative) of the oracle's 15th best
score (the k-th score of the rule: the diagonal block is not ranked). Each such block is a
near-tie; near-ties are counted and logged per workload (``TIE_LOG``, printed at the end of
the test session).

Cancellation near-ties. When the 15th score is itself close to zero -- its magnitude is
below ``CANCEL_RATIO`` of sum_i |q_i * kbar_i| / sqrt(d_I), the magnitude of the terms it is
summed from -- the relative window 1e-5 * |s15| is narrower than the fp32 rounding of any
score, and the order of those blocks is decided by rounding alone. Only in that case is a
differing block also accepted when it lies within 1e-5 of that term magnitude; such blocks
are counted separately. Rows whose 15th score is not near zero get the strict rule alone.
"""
from __future__ import annotations

import numpy as np

REL_TIE = 1e-5
CANCEL_RATIO = 0.1
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3

# Gradients of the main branch (dQ, dK, dV), relative to the reference's own magnitude (they are
# not O(1) like the outputs). Every gradient element is a sum of terms in which the kernel rounds
# one factor to bf16 (p for dV, dS = p (dP - D) for dQ and dK, whose D is formed from the
# forward's bf16 output): at most three roundings of 2^-9 relative each, accumulated in fp32.
# Random rounding errors of a sum stay near eps = 3 * 2^-9 of its typical magnitude, so the
# mean |err| is held to eps of the mean |ref| and the max |err| to 4 eps of the max |ref|.
GRAD_EPS = 3 * 2.0 ** -9
GRAD_REL_MEAN = GRAD_EPS
GRAD_REL_MAX = 4 * GRAD_EPS

# workload label -> counters (rows checked, rows differing, near-ties, cancellation near-ties)
TIE_LOG: dict = {}


def log_ties(label: str, rows: int, differing: int, near: int, cancel: int):
    e = TIE_LOG.setdefault(label, {"rows": 0, "differing_rows": 0, "near_ties": 0, "cancel_ties": 0})
    e["rows"] += int(rows)
    e["differing_rows"] += int(differing)
    e["near_ties"] += int(near)
    e["cancel_ties"] += int(cancel)


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
        elif (abs_scale is not None and abs(kth) < CANCEL_RATIO * abs_scale[b]
              and dlt <= REL_TIE * abs_scale[b]):
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


def sel_sorted_ok_rows(sel: np.ndarray) -> np.ndarray:
    """Vectorised sel_sorted_ok over rows of sel [n, k]: a bool per row."""
    sel = np.asarray(sel)
    valid = sel >= 0
    n = valid.sum(axis=1)
    prefix = np.arange(sel.shape[1])[None, :] < n[:, None]          # valid entries come first
    ascending = (np.diff(sel, axis=1) > 0) | ~prefix[:, 1:]
    return (valid == prefix).all(axis=1) & ascending.all(axis=1)


def error_metrics(gpu: np.ndarray, ref: np.ndarray):
    e = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


def assert_close_attention(gpu, ref, what=""):
    mx, mn = error_metrics(gpu, ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS_TOL, f"{what}: max abs err {mx:.3e} > {MAX_ABS_TOL}"
    assert mn <= MEAN_ABS_TOL, f"{what}: mean abs err {mn:.3e} > {MEAN_ABS_TOL}"
    return mx, mn


def assert_close_gradient(gpu, ref, what=""):
    """A gradient against the fp64 reference: mean |err| <= GRAD_REL_MEAN * mean |ref| and
    max |err| <= GRAD_REL_MAX * max |ref|."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(gpu).all(), f"{what}: non-finite gradient"
    e = np.abs(gpu - ref)
    mean_ref, max_ref = float(np.abs(ref).mean()), float(np.abs(ref).max())
    assert e.mean() <= GRAD_REL_MEAN * mean_ref, f"{what}: mean |err| {e.mean():.3e} > {GRAD_REL_MEAN:.2e} x {mean_ref:.3e}"
    assert e.max() <= GRAD_REL_MAX * max_ref, f"{what}: max |err| {e.max():.3e} > {GRAD_REL_MAX:.2e} x {max_ref:.3e}"
    return float(e.mean() / max(mean_ref, 1e-300)), float(e.max() / max(max_ref, 1e-300))
