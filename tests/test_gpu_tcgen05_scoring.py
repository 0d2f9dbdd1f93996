"""The tcgen05 (fifth-generation tensor core) top-k scoring kernel, selected with
TSD_SCORE_KERNEL=tcgen05, against the oracle (needs a B200).

Same checks as the default scoring kernel: every list of a small paged workload under the
top-k band rule (bf16 and fp32 queries -- the fp32 path adds the bf16 remainder MMAs), and the
exact-tie lists index for index.
"""

import math

import numpy as np
import pytest

import oracle
import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT
from tests import test_gpu_topk_ties as TIES

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
SMALL = W.DecodeConfig(name="small", batch=3, num_q_heads=8, num_kv_heads=2, seq_len=6000, tokens_per_seq=2,
                       ks=(100,), planted=True, causal=True)
SMALL_LENS = [6000, 300, 2500]


@pytest.fixture(autouse=True)
def tcgen05_scoring(monkeypatch):
    monkeypatch.setenv("TSD_SCORE_KERNEL", "tcgen05")
    yield


@pytest.mark.parametrize("q_f32", [False, True])
def test_tcgen05_topk_matches_oracle(q_f32):
    import torch
    w = W.make_workload(SMALL, seed=17, seq_lens=SMALL_LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=SMALL.max_seq_len, page_table=dw.page_table)
    q = dw.q.float() if q_f32 else dw.q
    queries = tsd.Queries(q, q_indptr=dw.q_indptr, max_tokens_per_seq=2, causal=True, sm_scale=SM_SCALE)
    inp = PT.OracleInputs(w)
    pairs = [(t, h) for t in range(len(w.kv_len)) for h in range(SMALL.num_q_heads)]
    for k in (1, 100, 400):
        idx, cnt = tsd.topk_select(cache, queries, k)
        torch.cuda.synchronize()
        stats = PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), w.k_per_token(k), pairs)
        assert stats["lists"] == len(pairs)
    assert tsd.read_device_status() == 0


@pytest.mark.parametrize("n_distinct", [2, 200])
def test_tcgen05_topk_ties(n_distinct):
    TIES.test_topk_ties_go_to_lower_indices(n_distinct)
