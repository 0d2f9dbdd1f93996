"""Acceptance rules for comparing a GPU result with the oracle (test infrastructure).

The rules are the ones the benchmark spec fixes for this path:
* top-k: the returned set must equal the exact top-k set (ties to the lower
  token index) except at tokens whose score lies within a relative band
  ``rel_band * |s_k|`` of the k-th score s_k (the GPU scores in float32, the
  oracle exactly); the counts must match.
* decode output: max-abs and relative-L2 error against the float64 result.
"""

from __future__ import annotations

import numpy as np

from .attention import exact_topk


def topk_sets_agree(gpu_list, scores, k: int, rel_band: float = 1e-4):
    """Check one GPU top-k list against the exact selection.

    gpu_list: the GPU's int32 list for one (query, head), length k_max, valid
    entries ascending then -1 padding.  scores: exact scores of tokens 0..L-1.
    Returns (ok: bool, reason: str).
    """
    s = np.asarray(scores, dtype=np.float64)
    L = s.shape[0]
    g = np.asarray(gpu_list, dtype=np.int64)
    n = min(k, L)
    valid = g[g >= 0]
    if valid.size != n:
        return False, f"count {valid.size} != {n}"
    if np.any(g[n:] != -1):
        return False, "padding after the valid entries is not all -1"
    if np.any(g[:n] < 0):
        return False, "-1 inside the valid prefix"
    if np.any(valid >= L):
        return False, "index out of range"
    if np.any(np.diff(valid) <= 0):
        return False, "entries not strictly ascending"
    ref = exact_topk(s, k)
    if n == 0:
        return True, ""
    sk = np.sort(s)[::-1][n - 1]
    band = rel_band * abs(sk)
    diff = np.setxor1d(ref, valid)
    bad = diff[np.abs(s[diff] - sk) > band]
    if bad.size:
        return False, f"{bad.size} tokens outside the band differ (e.g. {bad[:5].tolist()})"
    return True, ""


def output_errors(out, ref):
    """(max_abs, rel_l2) of `out` against the float64 reference `ref`."""
    o = np.asarray(out, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    d = o - r
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(d) / nr) if nr > 0 else float(np.linalg.norm(d))
    return max_abs, rel
