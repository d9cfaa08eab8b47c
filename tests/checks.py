"""Parity checks: compare a candidate result (normally the CUDA path's) with
the oracle, the way the DSA page (§3.1, tie discussion after eq. (18))
says a selection should be compared: first the cut-off value, then the set
strictly above it, then how many of the tied entries were returned.

Integer-valued workloads have exact fp32 scores, so there the index sets
must be identical (ties broken toward the lower position on both sides).
"""

from __future__ import annotations

import numpy as np

import oracle as O


def row_structure_errors(row, t: int, k: int) -> list:
    """Valid entries first (exactly min(k, t+1) of them), then -1 padding;
    every valid entry is a distinct position in [0, t]."""
    row = np.asarray(row, dtype=np.int64)
    m = min(k, t + 1)
    errs = []
    if row.shape != (k,):
        return [f"row shape {row.shape} != ({k},)"]
    valid, pad = row[:m], row[m:]
    if np.any(pad != -1):
        errs.append(f"t={t}: padding slots hold {pad[pad != -1][:4].tolist()}")
    if np.any(valid < 0) or np.any(valid > t):
        bad = valid[(valid < 0) | (valid > t)]
        errs.append(f"t={t}: {bad.size} valid slots out of [0,{t}]: {bad[:4].tolist()}")
    if np.unique(valid).size != valid.size:
        errs.append(f"t={t}: duplicate positions")
    return errs


def topk_exact_errors(cand_row, oracle_row, t: int, k: int) -> list:
    """Bit-exact comparison of index sets (slot order is free)."""
    errs = row_structure_errors(cand_row, t, k)
    m = min(k, t + 1)
    a = np.sort(np.asarray(cand_row, dtype=np.int64)[:m])
    b = np.sort(np.asarray(oracle_row, dtype=np.int64)[:m])
    if not np.array_equal(a, b):
        diff = np.setxor1d(a, b)
        errs.append(f"t={t}: index sets differ in {diff.size} positions, e.g. {diff[:6].tolist()}")
    return errs


def topk_tolerant_errors(cand_row, oracle_scores_row, t: int, k: int, rel: float = 1e-3):
    """Tolerance-aware comparison for float workloads.

    With tau the oracle's score at rank min(k, t+1) and
    tol = rel * max(|tau|, rel * max_s |I[s]|):
      * every selected position has oracle score >= tau - tol;
      * every position with oracle score > tau + tol is selected.
    Returns (errors, stats) with stats = overlap with the oracle set and the
    cut-off margin Delta_k of eq. (18).
    """
    errs = row_structure_errors(cand_row, t, k)
    s = np.asarray(oracle_scores_row, dtype=np.float64)[: t + 1] + 0.0
    st = O.selection_stats_row(s, t, k)
    m = min(k, t + 1)
    tol = rel * max(abs(st["tau"]), rel * st["max_abs"])
    sel = np.asarray(cand_row, dtype=np.int64)[:m]
    sel = sel[(sel >= 0) & (sel <= t)]
    low = sel[s[sel] < st["tau"] - tol]
    if low.size:
        errs.append(f"t={t}: {low.size} selected below tau-tol (tau={st['tau']:.6g}, "
                    f"worst={s[low].min():.6g})")
    must = np.nonzero(s > st["tau"] + tol)[0]
    missing = np.setdiff1d(must, sel)
    if missing.size:
        errs.append(f"t={t}: {missing.size} positions above tau+tol not selected")
    ref = O.causal_topk_row(s, t, k)[:m]
    overlap = np.intersect1d(ref, sel).size / m
    return errs, {"overlap": overlap, "margin": st["margin"], "tau": st["tau"]}


def close_errors(cand, ref, atol: float, rtol: float, what: str = "") -> list:
    """Elementwise |cand - ref| <= atol + rtol * |ref| (NaN/inf must match)."""
    c = np.asarray(cand, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if c.shape != r.shape:
        return [f"{what}: shape {c.shape} != {r.shape}"]
    both_inf = np.isinf(c) & np.isinf(r) & (np.sign(c) == np.sign(r))
    with np.errstate(invalid="ignore"):
        bad = ~(np.abs(c - r) <= atol + rtol * np.abs(r)) & ~both_inf
    if np.any(bad):
        i = np.unravel_index(np.argmax(np.where(bad, np.abs(c - r), -1)), c.shape)
        return [f"{what}: {int(bad.sum())} of {c.size} elements out of tolerance; worst at {i}: "
                f"{c[i]!r} vs {r[i]!r}"]
    return []
