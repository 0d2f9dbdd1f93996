"""CPU oracle for context-sparse decode attention (test infrastructure only).

This package is the slow, plain definition that the CUDA path is checked
against.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it; the library never does, and it imports nothing
from the library.  Everything is numpy in float64.

What it computes follows "Inference Time Context Sparsity: Illusion or
Opportunity?" (gist.science technical summary, section 2 "Oracle Top-K" and
"Hardware implementation"; section 3.C "bandwidth efficiency"):

* ``attention_scores``: s_i = sum_d q_d K_{i,d}, exact in float64 for bf16 inputs.
* ``exact_topk``: the exact top-k tokens of one (query, head) -- the pages'
  "Oracle Top-K" -- with ties going to the lower token index; returned in
  ascending token order.
* ``sparse_attention``: softmax attention restricted to a supplied index list
  (one term per list entry), giving the output row and its log-sum-exp.
* ``dense_attention``: the same over every visible token (the dense-decode
  baseline whose O(N d) traffic sparse decoding reduces to O(k d)).
* ``channel_importance``, ``choose_channels``, ``label_scores`` (``label.py``): the
  Double-Sparsity-style approximate indexer the pages use to price indexing (section
  3.C): a few "label" channels per kv head chosen by magnitude, approximate scores over
  them; its selection is ``exact_topk`` of those scores.
* ``floyd_sample``, ``stochastic_select``, ``weighted_attention`` (``vattention.py``): the
  vAttention-style stochastic selection the pages evaluate (section 2): exact top-k plus a
  uniform sample of the other tokens, each sample weighted by |rest| / m.
* ``topk_sets_agree``: the acceptance rule for a GPU top-k set (exact set
  equality except for tokens whose score is within a relative band of the
  k-th score).

Readings where the pages are silent (the pages print no formula, tie rule or
precision) are listed in the header of each function.
"""

from .attention import (  # noqa: F401
    attention_scores,
    dense_attention,
    exact_topk,
    from_bf16_bits,
    sparse_attention,
)
from .compare import (  # noqa: F401
    bf16_half_ulp,
    elementwise_bar,
    output_errors,
    output_within,
    topk_sets_agree,
)
from .label import channel_importance, choose_channels, label_scores  # noqa: F401
from .vattention import floyd_sample, stochastic_select, weighted_attention  # noqa: F401
