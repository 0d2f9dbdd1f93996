"""Acceptance rules for comparing a GPU result with the oracle (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU legs use this module.
The rules follow the bars the build is held to for this path:
* top-k: the returned set must equal the exact top-k set (ties to the lower
  token index) except at tokens whose score lies within a relative band
  ``rel_band * |s_k|`` of the k-th score s_k (the GPU scores in float32, the
  oracle exactly); the counts must match.
* decode output: max-abs and relative-L2 error against the float64 result.  For
  bf16 outputs the max-abs bar is 5e-3 wherever a bf16 value can meet it; where
  bf16 rounding alone exceeds it (|o| >= 2, half an ulp >= 2^-7), the bar is that
  half ulp plus the float32 evaluation's own error, budgeted at 1e-4 |o| -- the
  same relative allowance the top-k rule grants float32 scores.
"""

from __future__ import annotations

import numpy as np

from .attention import exact_topk

FP32_EVAL_REL = 1e-4   # relative error budget of a float32 evaluation before bf16 rounding


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


def bf16_half_ulp(x) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x|: bf16 keeps 8 significant bits, so the
    spacing in [2^e, 2^(e+1)) is 2^(e-7) and the worst rounding error half of it."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 8)


def elementwise_bar(ref, max_abs: float, bf16_rounded: bool) -> np.ndarray:
    """Per-element max-abs bar for an output against the float64 result `ref`.

    float32 outputs: `max_abs` everywhere.  bf16 outputs: max(max_abs, half a bf16 ulp of
    ref + FP32_EVAL_REL |ref|) -- `max_abs` itself wherever that is attainable."""
    r = np.asarray(ref, dtype=np.float64)
    if not bf16_rounded:
        return np.full(r.shape, float(max_abs))
    return np.maximum(float(max_abs), bf16_half_ulp(r) + FP32_EVAL_REL * np.abs(r))


def output_within(out, ref, max_abs: float, rel_l2: float, bf16_rounded: bool):
    """Apply both output bars: every element within `elementwise_bar`, and the relative L2
    error of the whole block at most `rel_l2`.  Returns (ok, reason)."""
    o = np.asarray(out, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if o.shape != r.shape:
        return False, f"shape {o.shape} != {r.shape}"
    if not np.all(np.isfinite(o)):
        return False, "non-finite output"
    excess = np.abs(o - r) - elementwise_bar(r, max_abs, bf16_rounded)
    if excess.size and np.max(excess) > 0:
        i = np.unravel_index(int(np.argmax(excess)), excess.shape)
        return False, (f"element {tuple(int(x) for x in i)}: {o[i]!r} vs {r[i]!r} exceeds the bar by "
                       f"{float(excess[i]):.3g}")
    _, rel = output_errors(o, r)
    if rel > rel_l2:
        return False, f"rel-L2 {rel:.3g} > {rel_l2}"
    return True, ""
