"""Context-parallel decode over a token-sharded cache, its P ranks run one after another on one
GPU (needs a B200).

The exchange between ranks is a stack of their tensors, in rank order, as an all-gather would
leave it.  The ranks' kernels never wait on one another, so running them in sequence is the
same computation.  Checks:
* the global top-k rebuilt from the ranks' kept entries equals the single-GPU top-k of the
  whole cache, index for index (each score is the same fp32 number either way, and the tie
  rule is the same);
* the merged output equals the single-GPU sparse decode over those lists (fp32), and the
  oracle's attention over the exact top-k where the lists agree with it;
* the shard views cover each sequence exactly once.
"""

import math

import numpy as np
import pytest

import oracle
import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import context_parallel as CP
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
CFG = W.DecodeConfig(name="cp", batch=4, num_q_heads=8, num_kv_heads=2, seq_len=20000, ks=(300,), planted=True)
LENS = [20000, 7000, 1500, 12345]


@pytest.fixture(scope="module")
def setup():
    w = W.make_workload(CFG, seed=13, seq_lens=LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=CFG.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, sm_scale=SM_SCALE)
    return w, cache, queries, PT.OracleInputs(w)


@pytest.mark.parametrize("P", [2, 3, 4])
def test_context_parallel_matches_single_gpu(setup, P):
    import torch
    w, cache, queries, inp = setup
    k = 300
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    S = CP.shard_length(cache.max_seq_len, P, 16)
    shards = [CP.shard_view(cache, r, P) for r in range(P)]
    lens = torch.stack([s.seq_lens for s in shards]).cpu().numpy()
    assert np.array_equal(lens.sum(axis=0), np.array(LENS))          # every token in exactly one shard
    # 1. local top-k with scores on each rank; 2. rank-major "all-gather"
    cands = [tsd.topk_select(s, queries, k, with_scores=True) for s in shards]
    cand_idx = torch.stack([c[0] for c in cands])
    cand_sc = torch.stack([c[1] for c in cands])
    # 3. each rank keeps its part of the global top-k; 4. partial decode on its shard
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mine = [CP.cp_merge_select(cand_idx, cand_sc, k, r, status=status) for r in range(P)]
    parts = [tsd.sparse_decode(s, queries, m, out_dtype=torch.float32) for s, m in zip(shards, mine)]
    # 5. merge
    out, lse = CP.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
                                 out_dtype=torch.float32)
    # single GPU
    ref_idx, _ = tsd.topk_select(cache, queries, k)
    ref_out, ref_lse = tsd.sparse_decode(cache, queries, ref_idx, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    glob = np.full((T, Hq, k), -1, dtype=np.int64)
    mine_np = [m.cpu().numpy() for m in mine]
    for t in range(T):
        for h in range(Hq):
            sel = np.concatenate([mine_np[r][t, h][mine_np[r][t, h] >= 0] + r * S for r in range(P)])
            glob[t, h, :sel.size] = sel
    assert np.array_equal(glob, ref_idx.cpu().numpy().astype(np.int64))
    o, ro = out.cpu().numpy(), ref_out.cpu().numpy()
    err, rel = oracle.output_errors(o.reshape(-1), ro.reshape(-1))
    assert err <= PT.F32_MAX_ABS and rel <= PT.F32_REL_L2, (err, rel)
    assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=PT.LSE_ABS, rtol=0)
    # and the oracle on the lists that equal its exact top-k
    for t in range(T):
        for h in range(Hq):
            exact = inp.topk(t, h, k)
            if np.array_equal(glob[t, h][:exact.size], exact):
                ro_, rl_ = inp.attend(t, h, exact, SM_SCALE)
                e, r_ = oracle.output_errors(o[t, h], ro_)
                assert e <= PT.F32_MAX_ABS and r_ <= PT.F32_REL_L2
    assert tsd.read_device_status() == 0


def test_merge_partials_edge_cases():
    """Empty parts (-inf lse) drop out; all-empty rows give 0 and -inf."""
    import torch
    P, T, Hq = 3, 2, 2
    outs = torch.randn((P, T, Hq, 128), device="cuda")
    lses = torch.randn((P, T, Hq), device="cuda")
    lses[1] = float("-inf")
    lses[:, 1, 1] = float("-inf")
    out, lse = CP.merge_partials(outs, lses, out_dtype=torch.float32)
    torch.cuda.synchronize()
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    on, ln = outs.cpu().numpy().astype(np.float64), lses.cpu().numpy().astype(np.float64)
    for t in range(T):
        for h in range(Hq):
            ls = ln[:, t, h]
            if np.all(np.isinf(ls)):
                assert np.all(o[t, h] == 0) and np.isinf(l[t, h]) and l[t, h] < 0
                continue
            m = np.max(ls[np.isfinite(ls)])
            wts = np.where(np.isfinite(ls), np.exp(ls - m), 0.0)
            ref = (wts[:, None] * on[:, t, h]).sum(axis=0) / wts.sum()
            assert np.allclose(o[t, h], ref, rtol=1e-5, atol=1e-6)
            assert abs(l[t, h] - (m + np.log(wts.sum()))) < 1e-5
