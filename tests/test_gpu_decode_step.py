"""tsd_decode_step -- exact top-k then sparse decode on one workspace -- against the oracle.

The step is captured into one CUDA graph and replayed; its index lists must pass the top-k
rule against the oracle's exact selection, and wherever a list equals the oracle's own list
exactly, its output must match the oracle's attention over that list.  The step must also be
bit-identical to the two calls made one after the other (tsd_topk_select, then
tsd_sparse_decode), since it runs the same kernels on the same plan.
"""

import math

import numpy as np
import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
SMALL = W.DecodeConfig(name="step_small", batch=3, num_q_heads=8, num_kv_heads=2, seq_len=6000, tokens_per_seq=2,
                       ks=(100,), planted=True, causal=True)


def _setup(cfg, lens=None, seed=0):
    w = W.make_workload(cfg, seed=seed, seq_lens=lens)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=cfg.max_seq_len,
                        page_table=None if cfg.layout == "contiguous" else dw.page_table)
    multi = cfg.tokens_per_seq > 1
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=cfg.causal, sm_scale=SM_SCALE)
    return w, cache, queries


def _graph_step(cache, queries, k_max, kpt, out_dtype):
    """decode_step captured once into a CUDA graph, replayed twice; returns its outputs."""
    import torch
    T, Hq = int(queries.q.shape[0]), int(queries.q.shape[1])
    ws = tsd.Workspace(cache.device)
    idx = torch.empty((T, Hq, k_max), dtype=torch.int32, device="cuda")
    cnt = torch.empty((T, Hq), dtype=torch.int32, device="cuda")
    out = torch.empty((T, Hq, 128), dtype=out_dtype, device="cuda")
    lse = torch.empty((T, Hq), dtype=torch.float32, device="cuda")

    def step():
        tsd.decode_step(cache, queries, k_max, k_per_token=kpt, out_idx=idx, out_count=cnt, out=out, lse=lse,
                        workspace=ws)

    step()   # sizes the workspace outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        out.fill_(float("nan"))
        g.replay()
    torch.cuda.synchronize()
    assert tsd.read_device_status(ws) == 0
    del g
    return idx, cnt, out, lse


def _check(w, cache, queries, k, pairs, out_dtype):
    import torch
    inp = PT.OracleInputs(w)
    kpt = w.k_per_token(k)
    k_max = int(kpt.max())
    kpt_dev = None if k is not None else torch.from_numpy(kpt).cuda()
    idx, cnt, out, lse = _graph_step(cache, queries, k_max, kpt_dev, out_dtype)
    gidx = idx.cpu().numpy()
    PT.check_topk(inp, gidx, cnt.cpu().numpy(), kpt, pairs)
    # the same two calls one after the other give the same bits
    i2, c2 = tsd.topk_select(cache, queries, k_max, k_per_token=kpt_dev)
    o2, l2 = tsd.sparse_decode(cache, queries, i2, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(i2, idx) and torch.equal(c2, cnt)
    assert torch.equal(o2, out) and torch.equal(l2, lse)
    # the output against the oracle wherever the step's list is the oracle's own list
    oidx = np.full_like(gidx, -1)
    same = []
    for t, h in pairs:
        ref = inp.topk(t, h, int(kpt[t]))
        oidx[t, h, :ref.size] = ref
        if np.array_equal(gidx[t, h], oidx[t, h]):
            same.append((t, h))
    assert len(same) >= 0.9 * len(pairs)
    PT.check_decode(inp, oidx, PT.bf16_to_np(out), lse.cpu().numpy(), same, SM_SCALE,
                    out_is_bf16=out_dtype == torch.bfloat16)
    return len(same)


def test_step_small_all_lists_fp32_and_bf16():
    import torch
    w, cache, queries = _setup(SMALL, lens=[6000, 300, 2500], seed=1)
    pairs = [(t, h) for t in range(len(w.kv_len)) for h in range(SMALL.num_q_heads)]
    for odt in (torch.float32, torch.bfloat16):
        _check(w, cache, queries, 100, pairs, odt)


def test_step_small_per_token_k():
    """k per token (ceil(0.02 kv_len), as the ragged workload asks) through k_per_token."""
    import torch
    cfg = W.DecodeConfig(name="step_ragged_small", batch=4, num_q_heads=8, num_kv_heads=2,
                         seq_len_range=(3000, 9000), tokens_per_seq=4, k_frac_ceil=0.02, planted=True, causal=True)
    w, cache, queries = _setup(cfg, seed=2)
    pairs = [(t, h) for t in range(len(w.kv_len)) for h in range(cfg.num_q_heads)]
    _check(w, cache, queries, None, pairs, torch.float32)


def test_step_without_caller_index_buffer():
    """out_idx = NULL keeps the lists inside the workspace; the output is unchanged."""
    import torch
    w, cache, queries = _setup(SMALL, lens=[6000, 300, 2500], seed=1)
    ref_out, ref_lse, _ = tsd.decode_step(cache, queries, 100, out_idx=torch.empty((6, 8, 100), dtype=torch.int32,
                                                                                    device="cuda"))
    out, lse, idx = tsd.decode_step(cache, queries, 100)
    torch.cuda.synchronize()
    assert idx is None
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_step_llama3_8b_sampled():
    import torch
    w, cache, queries = _setup(W.CONFIGS["llama3_8b"], seed=0)
    pairs = PT.sample_pairs(w, 8, full_seqs=(0,), seed=3)
    _check(w, cache, queries, 655, pairs, torch.bfloat16)


@pytest.mark.parametrize("per_token", [False, True])
def test_step_with_the_candidate_filter_forced(monkeypatch, per_token):
    """The step with the exact indexer's candidate filter forced on (TSD_TOPK_FILTER=1): its
    pre-pass arrival counters, candidate counters and queue must be left zero by every replay,
    so that the second replay of the graph agrees with the oracle as the first did."""
    import torch
    monkeypatch.setenv("TSD_TOPK_FILTER", "1")
    if per_token:
        cfg = W.DecodeConfig(name="step_ragged_small", batch=4, num_q_heads=8, num_kv_heads=2,
                             seq_len_range=(3000, 20000), tokens_per_seq=4, k_frac_ceil=0.02, planted=True,
                             causal=True)
        w, cache, queries = _setup(cfg, seed=4)
        k = None
    else:
        w, cache, queries = _setup(SMALL, lens=[6000, 300, 2500], seed=1)
        k = 100
    kpt = w.k_per_token(k)
    assert tsd.topk_select_plan(cache, queries, int(kpt.max()))["filtered"]
    pairs = [(t, h) for t in range(len(w.kv_len)) for h in range(w.cfg.num_q_heads)]
    _check(w, cache, queries, k, pairs, torch.float32)


def test_step_ragged_8_sampled():
    """The ragged batch with 8 sequences, where the filter runs by default (537 MB of score rows
    would not stay in L2)."""
    import torch
    w, cache, queries = _setup(W.CONFIGS["ragged_8"], seed=0)
    kpt = w.k_per_token(None)
    assert tsd.topk_select_plan(cache, queries, int(kpt.max()))["filtered"]
    pairs = PT.sample_pairs(w, 8, full_seqs=(0,), seed=5)
    _check(w, cache, queries, None, pairs, torch.bfloat16)
