"""The exact indexer's candidate filter, each of its paths against the oracle (needs a B200).

With bf16 queries and a small enough k the exact indexer scores a sample of every list first,
turns it into a threshold, and has the scoring kernel append the scores at or above it instead
of writing score rows; the selection then works on those candidates alone.  A list the
candidates cannot serve has its row recomputed by the selection.  The result must be the exact
top-k in every case ("Oracle Top-K", section 2 of the pages' summary).  The paths:

- TSD_TOPK_FILTER=1, the filter forced on (by default it runs only where the score rows would
  not stay in L2, which this small case does not reach), on lists up to the candidate buffer's
  size (every score a candidate) and on longer lists (a sampled threshold), with per-token k
  including 0, 1, k >= kv_len;
- TSD_TOPK_FILTER=rescore, which disables every threshold so that every list takes the
  recomputation;
- TSD_TOPK_FILTER=0, the unfiltered form over score rows.

The filtered and unfiltered forms score every token with the same tensor-core tile, so the lists
they select must agree index for index; the recomputed scores round differently, so that path
is held to the oracle's band only.
"""

import math

import numpy as np
import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
CFG = W.DecodeConfig(name="filter_mix", batch=5, num_q_heads=8, num_kv_heads=2, seq_len=40000, tokens_per_seq=2,
                     ks=(300,), planted=True, causal=True)
LENS = [40000, 9000, 6000, 300, 21001]   # above, around and below the 8192-entry candidate buffer


@pytest.fixture(scope="module")
def case():
    w = W.make_workload(CFG, seed=21, seq_lens=LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=CFG.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr, max_tokens_per_seq=CFG.tokens_per_seq, causal=True,
                          sm_scale=SM_SCALE)
    return w, cache, queries, PT.OracleInputs(w)


def _pairs(w):
    return [(t, h) for t in range(len(w.kv_len)) for h in range(w.cfg.num_q_heads)]


def _select(monkeypatch, mode, cache, queries, k_max, kpt):
    import torch
    if mode is None:
        monkeypatch.delenv("TSD_TOPK_FILTER", raising=False)
    else:
        monkeypatch.setenv("TSD_TOPK_FILTER", mode)
    idx, cnt = tsd.topk_select(cache, queries, k_max,
                               k_per_token=None if kpt is None else torch.from_numpy(kpt).cuda())
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("per_token", [False, True])
def test_filtered_paths_agree_with_the_oracle(monkeypatch, case, per_token):
    w, cache, queries, inp = case
    T = len(w.kv_len)
    if per_token:   # k = 0, 1, k >= kv_len (the 300-token sequence's tokens 6 and 7), and 2%
        kpt = np.array([int(math.ceil(0.02 * L)) for L in w.kv_len], dtype=np.int32)
        kpt[1], kpt[2], kpt[6], kpt[7] = 0, 1, 299, 400
        k_max = int(kpt.max())
        want = np.minimum(kpt, k_max)
    else:
        kpt, k_max = None, 300
        want = np.full(T, 300, dtype=np.int32)
    runs = {}
    for mode in ("1", "rescore", "0"):
        idx, cnt = _select(monkeypatch, mode, cache, queries, k_max, kpt)
        PT.check_topk(inp, idx, cnt, want, _pairs(w))
        runs[mode] = idx
    assert np.array_equal(runs["1"], runs["0"])
    assert tsd.read_device_status() == 0


@pytest.mark.parametrize("mode", ["1", "rescore"])
def test_filter_keeps_the_lowest_tied_indices(monkeypatch, case, mode):
    """Equal scores straddling the k-th place: a query of zeros gives every token the score 0,
    so every list is one tie group, and the rule keeps the lowest indices.  Lists up to 8192
    tokens take every score as a candidate and resolve the tie there; longer ones overflow the
    candidate buffer and take the recomputed row."""
    import torch
    w, cache, _, inp = case
    q0 = torch.zeros((len(w.kv_len), CFG.num_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    queries = tsd.Queries(q0, q_indptr=torch.from_numpy(w.q_indptr).cuda(), max_tokens_per_seq=CFG.tokens_per_seq, causal=True,
                          sm_scale=SM_SCALE)
    monkeypatch.setenv("TSD_TOPK_FILTER", mode)
    idx, cnt = tsd.topk_select(cache, queries, 50)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    for t, h in _pairs(w):
        n = min(50, int(w.kv_len[t]))
        assert np.array_equal(idx[t, h, :n], np.arange(n)), (t, h)
        assert (idx[t, h, n:] == -1).all()
    assert tsd.read_device_status() == 0
