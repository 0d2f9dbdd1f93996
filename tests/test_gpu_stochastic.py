"""vAttention-style stochastic selection and weighted sparse decode: CUDA path vs the oracle.

The top-k lists fed to the GPU are the oracle's, and the random words are drawn here by a
seeded numpy generator, so both sides sample from the same words: the GPU's index lists
must equal the oracle's exactly, its log-weights to fp32 rounding, and the weighted decode
must match the oracle's weighted attention within the fp32 output tolerance.
"""

import math

import numpy as np
import pytest

import oracle
import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
SMALL = W.DecodeConfig(name="small", batch=3, num_q_heads=8, num_kv_heads=2, seq_len=6000, tokens_per_seq=2,
                       ks=(100,), planted=True, causal=True)
SMALL_LENS = [6000, 300, 2500]


@pytest.fixture(scope="module")
def small():
    w = W.make_workload(SMALL, seed=5, seq_lens=SMALL_LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=SMALL.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr, max_tokens_per_seq=2, causal=True, sm_scale=SM_SCALE)
    return w, cache, queries, PT.OracleInputs(w)


def _oracle_topk(w, inp, k):
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    idx = np.full((T, Hq, k), -1, dtype=np.int32)
    for t in range(T):
        for h in range(Hq):
            sel = inp.topk(t, h, k)
            idx[t, h, :sel.size] = sel
    return idx


@pytest.mark.parametrize("k,m", [(100, 0), (100, 7), (50, 300), (20, 1024)])
def test_stochastic_select_and_weighted_decode(small, k, m):
    import torch
    w, cache, queries, inp = small
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    top = _oracle_topk(w, inp, k)
    u = np.random.default_rng(100 + m).integers(0, 2**32, size=(T, Hq, max(m, 1)), dtype=np.uint64)[:, :, :m]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gidx, glw = tsd.stochastic_select(cache, queries, torch.from_numpy(top).cuda(),
                                      torch.from_numpy(u.astype(np.int64)).cuda(), status=status)
    out, lse = tsd.sparse_decode(cache, queries, gidx, logw=glw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    gidx, glw = gidx.cpu().numpy(), glw.cpu().numpy()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    assert int(status.item()) == 0
    G = w.cfg.group
    for t in range(T):
        b, L = int(w.token_seq[t]), int(w.kv_len[t])
        for h in range(Hq):
            K, V = inp.kv(b, h // G)
            s = inp.scores(t, h)
            ridx, rlw = oracle.stochastic_select(s, k, m, u[t, h])
            n = ridx.size
            assert np.array_equal(gidx[t, h, :n], ridx), (k, m, t, h)
            assert np.all(gidx[t, h, n:] == -1)
            assert np.allclose(glw[t, h, :n], rlw, rtol=1e-6, atol=1e-6)
            ro, rl = oracle.weighted_attention(inp.q(t, h), K[:L], V[:L], ridx, rlw, SM_SCALE)
            err, rel = oracle.output_errors(out[t, h], ro)
            assert err <= PT.F32_MAX_ABS and rel <= PT.F32_REL_L2, (k, m, t, h, err, rel)
            assert abs(lse[t, h] - rl) <= PT.LSE_ABS
    assert tsd.read_device_status() == 0


def test_sampling_the_whole_rest_is_dense(small):
    import torch
    w, cache, queries, inp = small
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    top = _oracle_topk(w, inp, 10)
    m = 1024
    short = W.make_workload(SMALL, seed=5, seq_lens=SMALL_LENS)   # the 300-token sequence: rest < m
    u = np.random.default_rng(7).integers(0, 2**32, size=(T, Hq, m), dtype=np.uint64)
    gidx, glw = tsd.stochastic_select(cache, queries, torch.from_numpy(top).cuda(),
                                      torch.from_numpy(u.astype(np.int64)).cuda())
    out, lse = tsd.sparse_decode(cache, queries, gidx, logw=glw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for t in range(T):
        if int(short.token_seq[t]) != 1:
            continue
        for h in range(Hq):
            ro, _ = inp.dense(t, h, SM_SCALE)
            err, rel = oracle.output_errors(out[t, h], ro)
            assert err <= PT.F32_MAX_ABS and rel <= PT.F32_REL_L2


def test_bad_topk_list_is_flagged(small):
    import torch
    w, cache, queries, inp = small
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    top = _oracle_topk(w, inp, 16)
    top[0, 0, :2] = top[0, 0, 1::-1]          # not ascending
    u = np.zeros((T, Hq, 4), dtype=np.int64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tsd.stochastic_select(cache, queries, torch.from_numpy(top).cuda(), torch.from_numpy(u).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & tsd.DEV_BAD_INDEX
