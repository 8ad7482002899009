"""Shared test helpers: error metrics and top-k agreement (no method arithmetic)."""
from __future__ import annotations

import numpy as np


def rel_err(got, ref, floor_frac: float = 1.0) -> float:
    """max_i |g_i - r_i| / max(|r_i|, floor_frac * rms(r)).

    A plain max relative error is ill-conditioned for values near zero; the floor ties
    those to the scale of the whole output.  floor_frac = 1 is the metric the parity
    tests assert; smaller floors are reported alongside.
    """
    g = np.asarray(got, dtype=np.float64).reshape(-1)
    r = np.asarray(ref, dtype=np.float64).reshape(-1)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    den = np.maximum(np.abs(r), floor_frac * rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(g - r) / den))


def normwise_err(got, ref) -> float:
    """max_i |g_i - r_i| / max_i |r_i|: the max-norm relative error of the whole output."""
    g = np.asarray(got, dtype=np.float64).reshape(-1)
    r = np.asarray(ref, dtype=np.float64).reshape(-1)
    if r.size == 0:
        return 0.0
    den = float(np.max(np.abs(r)))
    return float(np.max(np.abs(g - r)) / (den if den > 0 else 1.0))


def check_close(got, ref, dtype: str, what: str = "") -> dict:
    """Parity bar for one output.

    bf16: normwise error <= 2e-2 (the stated tolerance, read as the max-norm relative
    error of the output vector) and the elementwise error, floored at the output's rms,
    <= 5e-2.  fp32: both <= 1e-4.  Returns the measured metrics (also the elementwise
    error with a 0.1*rms floor, for information)."""
    tol = 2e-2 if dtype == "bf16" else 1e-4
    tol_el = 5e-2 if dtype == "bf16" else 1e-4
    m = {"normwise": normwise_err(got, ref), "elementwise_rms_floor": rel_err(got, ref),
         "elementwise_0.1rms_floor": rel_err(got, ref, 0.1)}
    assert m["normwise"] <= tol and m["elementwise_rms_floor"] <= tol_el, (what, m)
    return m


def topk_agrees(got_idx, ref_scores, k: int, tol_abs: float) -> tuple[bool, str]:
    """GPU top-k against oracle scores.

    Position j must hold the oracle's j-th index whenever the oracle's j-th score is
    separated from both neighbours by more than tol_abs; elsewhere the GPU's index must
    still be a valid member of the tolerance band (its oracle score within tol_abs of
    the oracle's j-th score).
    """
    r = np.asarray(ref_scores, dtype=np.float64)
    order = np.lexsort((np.arange(len(r)), -r))
    ref_idx = order[:k]
    got_idx = np.asarray(got_idx)
    if len(got_idx) != len(ref_idx):
        return False, "length"
    if len(set(got_idx.tolist())) != len(got_idx):
        return False, "duplicate index"
    srt = r[order]
    for j in range(len(ref_idx)):
        gap_prev = srt[j - 1] - srt[j] if j > 0 else np.inf
        gap_next = srt[j] - srt[j + 1] if j + 1 < len(srt) else np.inf
        if min(gap_prev, gap_next) > tol_abs:
            if got_idx[j] != ref_idx[j]:
                return False, f"position {j}: got {got_idx[j]} want {ref_idx[j]}"
        elif abs(r[got_idx[j]] - srt[j]) > 2 * tol_abs:
            return False, f"position {j}: {got_idx[j]} outside the tolerance band"
    return True, "ok"
