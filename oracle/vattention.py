"""vAttention-style stochastic selection: plain float64 definitions.

Test infrastructure only (see the package header).  Source: "Inference Time Context
Sparsity: Illusion or Opportunity?", gist.science technical summary, section 2
("Stochastic indexing": vAttention is evaluated to see whether stochastic selection recovers
the quality that deterministic top-k loses on smaller models) and section 3.A (stochastic
versus deterministic).  The pages give neither the sampling scheme nor the estimator.
Readings:
* the deterministic part is the exact top-k S of the list (``exact_topk``);
* the rest R = [0, L) minus S is sampled uniformly without replacement, m tokens, by
  Floyd's algorithm (R. W. Floyd, "A sample of brilliance", CACM 1987) driven by random
  32-bit words supplied by the caller: step j (j = |R| - m .. |R| - 1) draws
  t = u_j mod (j + 1) and keeps t, or keeps j when t is already kept;
* each sampled token stands for |R| / m tokens of R: the softmax numerator and denominator
  weight it by w = |R| / m (the Horvitz-Thompson estimator of the sums over R), the top-k
  tokens by 1.
"""

from __future__ import annotations

import numpy as np

from .attention import exact_topk


def floyd_sample(n: int, m: int, u) -> np.ndarray:
    """m distinct ranks of [0, n), ascending, from the random words u[0..m) (Floyd's algorithm)."""
    m = max(0, min(int(m), int(n)))
    u = np.asarray(u, dtype=np.uint64)
    chosen = set()
    for step, j in enumerate(range(n - m, n)):
        t = int(u[step] % np.uint64(j + 1))
        chosen.add(j if t in chosen else t)
    return np.array(sorted(chosen), dtype=np.int64)


def stochastic_select(scores, k: int, m: int, u):
    """(index list ascending, log-weights) of top-k + m uniform samples of the rest.

    Log-weights are 0 for the top-k tokens and ln(|R| / m_eff) for the sampled ones, where
    m_eff = min(m, |R|)."""
    s = np.asarray(scores, dtype=np.float64)
    L = s.shape[0]
    top = exact_topk(s, k)
    rest = np.setdiff1d(np.arange(L), top)
    m_eff = min(int(m), rest.size)
    sampled = rest[floyd_sample(rest.size, m_eff, u)] if m_eff > 0 else np.zeros(0, dtype=np.int64)
    idx = np.concatenate([top, sampled])
    lw = np.concatenate([np.zeros(top.size), np.full(sampled.size, np.log(rest.size / m_eff) if m_eff else 0.0)])
    order = np.argsort(idx, kind="stable")
    return idx[order].astype(np.int64), lw[order]


def weighted_attention(q, K, V, idx, logw, sm_scale: float):
    """Softmax attention over the listed entries, entry i weighted by exp(logw_i):
    out = sum_i w_i e^{z_i} V_i / sum_i w_i e^{z_i}, lse = ln sum_i w_i e^{z_i}, z = sm_scale q.K."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    logw = np.asarray(logw, dtype=np.float64)
    keep = idx >= 0
    idx, logw = idx[keep], logw[keep]
    if idx.size == 0:
        return np.zeros(V.shape[1]), float("-inf")
    z = sm_scale * (K[idx] @ q) + logw
    mx = np.max(z)
    e = np.exp(z - mx)
    den = np.sum(e)
    return (e @ V[idx]) / den, float(mx + np.log(den))
