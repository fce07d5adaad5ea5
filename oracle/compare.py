"""Comparison rules between the CUDA path and the oracle (test
infrastructure).

* Floating-point outputs: max|got - ref| / max|ref| per tensor <= 1e-2 (bf16
  storage, float32 accumulation).
* Top-k index sets: let s_k be the oracle's k-th highest score of a row; the
  entries whose score lies within 1e-4 * max(|s_k|, 1e-30) of s_k form the
  tie zone.  Outside it the kept sets must be identical; inside it any choice
  of the right size is valid.  The output must list its indices ascending,
  padded with -1, all of them visible.
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-4
OUT_TOL = 1e-2


def max_abs_rel(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max() if ref.size else 0.0
    num = np.abs(got - ref).max() if ref.size else 0.0
    return float(num / den) if den > 0 else float(num)


def elem_rel(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3))) if ref.size else 0.0


def check_topk_row(got_row, ref_scores, k) -> str | None:
    """None if got_row is a valid top-k of ref_scores under the tie rule,
    else a description of the mismatch."""
    got_row = np.asarray(got_row, dtype=np.int64)
    n = ref_scores.shape[0]
    nk = min(k, n)
    if got_row.shape != (k,):
        return f"shape {got_row.shape}"
    sel = got_row[:nk]
    if np.any(got_row[nk:] != -1):
        return "padding is not -1"
    if nk and (np.any(sel < 0) or np.any(sel >= n)):
        return f"index out of range: {sel.min()}..{sel.max()} for {n} visible"
    if np.any(np.diff(sel) <= 0):
        return "indices not strictly ascending"
    if n <= k:
        return None if np.array_equal(sel, np.arange(n)) else "all visible entries must be kept"
    order = np.lexsort((np.arange(n), -ref_scores))
    s_k = ref_scores[order[k - 1]]
    tie = np.abs(ref_scores - s_k) <= TIE_REL * max(abs(s_k), 1e-30)
    ref_keep = np.zeros(n, bool)
    ref_keep[order[:k]] = True
    got_keep = np.zeros(n, bool)
    got_keep[sel] = True
    if np.any(ref_keep[~tie] != got_keep[~tie]):
        bad = np.flatnonzero((ref_keep != got_keep) & ~tie)
        return f"{bad.size} differences outside the tie zone (first {bad[:5]})"
    if got_keep[tie].sum() != ref_keep[tie].sum():
        return "wrong number of tie-zone entries"
    return None
