"""Plain float64 definitions of exact top-k selection and (sparse) decode attention.

Test infrastructure only (see the package header).  Source of each step:
"Inference Time Context Sparsity: Illusion or Opportunity?", gist.science
technical summary (Dutch, Spanish and Chinese versions), section 2
"Sparsiteitsmechanismen / Oracle Top-K" (exact selection of the top-k tokens)
and section 3.C (sparse decoding reads O(k d) instead of O(N d)); the
softmax-attention form itself is not printed on the pages and is taken as the
standard scaled dot-product attention.
"""

from __future__ import annotations

import numpy as np


def from_bf16_bits(bits) -> np.ndarray:
    """Exact float64 values of bf16 numbers stored as uint16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def attention_scores(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """s_i = sum_d q_d * K[i, d] in float64.

    q: [D]; K: [L, D].  For bf16 q and K every product is exact in float64;
    for moderate magnitudes (2^-8 <= |x| < 4, the bulk of N(0,1) data) the
    128-term sum is exact too, and otherwise it is within a few float64 ulps
    of the exact dot product -- far below float32 resolution.
    The selection ignores the softmax scale (a positive constant does not change
    the order); attention applies it.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    return K @ q


def exact_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Exact top-k ("Oracle Top-K", section 2 of the pages).

    Order the tokens 0..L-1 by (score descending, token index ascending), keep
    the first min(k, L), and return them in ascending token order (int64).
    Readings: ties go to the lower token index; -0.0 equals +0.0 (plain float
    comparison); k >= L keeps every token.
    """
    s = np.asarray(scores, dtype=np.float64)
    L = s.shape[0]
    n = max(0, min(int(k), L))
    idx = np.arange(L)
    # lexsort sorts by the last key first: primary -score ascending, then index.
    order = np.lexsort((idx, -s))
    return np.sort(order[:n]).astype(np.int64)


def sparse_attention(q, K, V, idx, sm_scale: float):
    """Softmax attention of one query row over the tokens of one index list.

    w_i = exp(sm_scale * s_i - max_j sm_scale * s_j) for each entry i of idx
    (every entry is a term, so a token listed twice counts twice), then
        out = sum_i w_i V_i / sum_i w_i,   lse = max_j sm_scale * s_j + ln sum_i w_i.
    An empty list gives out = 0 and lse = -inf.
    q: [D]; K, V: [L, D]; idx: entries of [0, L) (-1 entries are padding and skipped).
    Returns (out float64 [D], lse float).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64).reshape(-1)
    idx = idx[idx >= 0]
    D = V.shape[1]
    if idx.size == 0:
        return np.zeros(D, dtype=np.float64), float("-inf")
    z = sm_scale * (K[idx] @ q)
    m = np.max(z)
    w = np.exp(z - m)
    denom = np.sum(w)
    out = (w @ V[idx]) / denom
    return out, float(m + np.log(denom))


def dense_attention(q, K, V, sm_scale: float):
    """Dense decode attention: sparse_attention over every token 0..L-1."""
    L = np.asarray(K).shape[0]
    return sparse_attention(q, K, V, np.arange(L), sm_scale)
