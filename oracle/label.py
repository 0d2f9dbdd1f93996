"""Double-Sparsity-style approximate indexer: plain float64 definitions.

Test infrastructure only (see the package header).  Source: "Inference Time Context
Sparsity: Illusion or Opportunity?", gist.science technical summary, section 3.C
("Indexing overhead"): the pages price the indexer that chooses the k tokens by
simulating Double Sparsity in front of the sparse decode kernel, and report the net
speed-up including it.  Double Sparsity scores every token with only a few "label"
channels of the keys, chosen offline, and keeps the top k of those approximate scores.

The pages give neither the number of channels nor how they are chosen.  Readings:
* r channels per kv head (a multiple of 8; 16 by default);
* the importance of channel d for kv head g is the total magnitude of that channel's
  products over the calibration pairs: the sum, over sequences b, queries t of b, q heads
  h of group g and visible tokens i of b, of |q[t,h,d] * K[b,g,i,d]|;
* the r most important channels are kept, ties to the lower channel index, in ascending
  channel order;
* the approximate score of token i is s~_i = sum over kept channels d of q_d K_{i,d}, and
  the selection is the exact top-k of s~ (same tie rule as the exact indexer).
"""

from __future__ import annotations

import numpy as np


def channel_importance(Q, K) -> np.ndarray:
    """Per-channel sum of |Q[t, d] * K[i, d]| over every (query row t, key row i) pair.

    Q: [n, D] the queries of one (sequence, kv head) group; K: [L, D] its visible keys.
    Since every term is a product of two magnitudes, the double sum factors exactly into
    (sum_t |Q[t, d]|) * (sum_i |K[i, d]|), which is what is evaluated here.
    """
    Q = np.abs(np.asarray(Q, dtype=np.float64))
    K = np.abs(np.asarray(K, dtype=np.float64))
    return Q.sum(axis=0) * K.sum(axis=0)


def choose_channels(importance, r: int) -> np.ndarray:
    """The r most important channels (ties to the lower index), ascending (int64)."""
    imp = np.asarray(importance, dtype=np.float64)
    D = imp.shape[0]
    order = np.lexsort((np.arange(D), -imp))
    return np.sort(order[:max(0, min(int(r), D))]).astype(np.int64)


def label_scores(q, K, channels) -> np.ndarray:
    """s~_i = sum over d in channels of q_d K[i, d] (float64).  q: [D]; K: [L, D]."""
    c = np.asarray(channels, dtype=np.int64)
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    return K[:, c] @ q[c]
