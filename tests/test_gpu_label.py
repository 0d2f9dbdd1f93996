"""Label-channel (Double-Sparsity-style) indexer: CUDA path vs the oracle (needs a B200).

* Channel choice: the GPU's calibration against the oracle's importance and choice, equal
  except where two channels' exact importances are within 1e-5 (relative) at the r-th place.
* Label cache: a gather, compared bit for bit with the host's K rows at the channels.
* Approximate top-k: with channels the test draws itself (seeded, not the GPU's), the GPU
  list against the oracle's exact top-k of the label scores, under the top-k band rule.
* Pipeline: GPU label top-k, then GPU sparse decode, against the oracle's attention over the
  oracle's label top-k lists (for lists where the two selections agree).
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
    import torch
    w = W.make_workload(SMALL, seed=3, seq_lens=SMALL_LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=SMALL.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr, max_tokens_per_seq=2, causal=True, sm_scale=SM_SCALE)
    return w, dw, cache, queries, PT.OracleInputs(w)


def _test_channels(hkv: int, r: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(128, size=r, replace=False)) for _ in range(hkv)]).astype(np.int32)


def _oracle_importance(w, inp, g):
    G = w.cfg.group
    imp = np.zeros(128)
    for b in range(w.cfg.batch):
        K, _ = inp.kv(b, g)
        Q = np.stack([inp.q(t, h) for t in range(int(w.q_indptr[b]), int(w.q_indptr[b + 1]))
                      for h in range(g * G, (g + 1) * G)])
        imp += oracle.channel_importance(Q, K[:int(w.seq_lens[b])])
    return imp


@pytest.mark.parametrize("r", [8, 16, 32])
def test_label_channels_match_oracle(small, r):
    import torch
    w, dw, cache, queries, inp = small
    ch = tsd.label_channels(cache, queries, r)
    torch.cuda.synchronize()
    ch = ch.cpu().numpy()
    for g in range(w.cfg.num_kv_heads):
        imp = _oracle_importance(w, inp, g)
        ref = oracle.choose_channels(imp, r)
        got = ch[g]
        assert np.all(np.diff(got) > 0) and got.min() >= 0 and got.max() < 128
        diff = np.setxor1d(ref, got)
        if diff.size:
            pivot = np.sort(imp)[::-1][r - 1]
            assert np.all(np.abs(imp[diff] - pivot) <= 1e-5 * pivot), (g, diff)


def test_label_cache_is_the_channel_gather(small):
    import torch
    w, dw, cache, queries, inp = small
    chans = _test_channels(w.cfg.num_kv_heads, 16, seed=4)
    idx = tsd.label_cache_build(cache, torch.from_numpy(chans).cuda())
    torch.cuda.synchronize()
    lab = idx.label_k.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1, 16)
    rng = np.random.default_rng(5)
    for b in range(w.cfg.batch):
        for g in range(w.cfg.num_kv_heads):
            L = int(w.seq_lens[b])
            toks = np.unique(rng.integers(0, L, size=64))
            kb = w.logical_kv_bits(b, g, "k", toks)
            for j, i in enumerate(toks):
                row = w.physical_row(b, g, int(i))
                assert np.array_equal(lab[row], kb[j, chans[g]]), (b, g, int(i))


@pytest.mark.parametrize("r", [8, 16, 32])
def test_label_topk_matches_oracle(small, r):
    import torch
    w, dw, cache, queries, inp = small
    chans = _test_channels(w.cfg.num_kv_heads, r, seed=10 + r)
    index = tsd.label_cache_build(cache, torch.from_numpy(chans).cuda())
    G = w.cfg.group
    for k in (1, 100, 700):
        gidx, gcnt = tsd.topk_select_label(cache, index, queries, k)
        torch.cuda.synchronize()
        gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
        for t in range(len(w.kv_len)):
            b, L = int(w.token_seq[t]), int(w.kv_len[t])
            for h in range(w.cfg.num_q_heads):
                K, _ = inp.kv(b, h // G)
                s = oracle.label_scores(inp.q(t, h), K[:L], chans[h // G])
                ok, why = oracle.topk_sets_agree(gidx[t, h], s, k, PT.TOPK_BAND)
                assert ok, (r, k, t, h, why)
                assert int(gcnt[t, h]) == min(k, L)
    assert tsd.read_device_status() == 0


def test_label_pipeline_decode(small):
    import torch
    w, dw, cache, queries, inp = small
    chans = _test_channels(w.cfg.num_kv_heads, 16, seed=21)
    index = tsd.label_cache_build(cache, torch.from_numpy(chans).cuda())
    gidx, _ = tsd.topk_select_label(cache, index, queries, 100)
    out, lse = tsd.sparse_decode(cache, queries, gidx, out_dtype=torch.float32)
    torch.cuda.synchronize()
    gidx = gidx.cpu().numpy()
    G = w.cfg.group
    oidx = np.full_like(gidx, -1)
    same = []
    for t in range(len(w.kv_len)):
        b, L = int(w.token_seq[t]), int(w.kv_len[t])
        for h in range(w.cfg.num_q_heads):
            K, _ = inp.kv(b, h // G)
            sel = oracle.exact_topk(oracle.label_scores(inp.q(t, h), K[:L], chans[h // G]), 100)
            oidx[t, h, :sel.size] = sel
            if np.array_equal(gidx[t, h], oidx[t, h]):
                same.append((t, h))
    assert len(same) >= 0.95 * gidx.shape[0] * gidx.shape[1]
    PT.check_decode(inp, oidx, out.cpu().numpy(), lse.cpu().numpy(), same, SM_SCALE, out_is_bf16=False)


ONE_TOKEN = W.DecodeConfig(name="label_one_token", batch=3, num_q_heads=8, num_kv_heads=2, seq_len=20000,
                           tokens_per_seq=1, ks=(200,), planted=True, causal=True)


@pytest.mark.parametrize("cfg_lens", [(SMALL, SMALL_LENS, 3), (ONE_TOKEN, [20000, 9000, 3000], 4)],
                         ids=["8_lists_per_group", "4_lists_per_group"])
@pytest.mark.parametrize("r", [8, 16])
def test_label_topk_candidate_filter(monkeypatch, cfg_lens, r):
    """The label indexer's candidate filter (forced on with TSD_TOPK_FILTER=1), its row
    recomputation (TSD_TOPK_FILTER=rescore) and the row form (=0), each against the oracle's
    exact top-k of the label scores; the filtered and row forms score every token the same way,
    so their lists must agree index for index.  Groups of 4 lists take the scoring kernel that
    keeps the queries in registers, groups of 8 the general one."""
    import torch
    cfg, lens, seed = cfg_lens
    w = W.make_workload(cfg, seed=seed, seq_lens=lens)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=cfg.max_seq_len, page_table=dw.page_table)
    multi = cfg.tokens_per_seq > 1
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=True, sm_scale=SM_SCALE)
    inp = PT.OracleInputs(w)
    chans = _test_channels(cfg.num_kv_heads, r, seed=30 + r)
    index = tsd.label_cache_build(cache, torch.from_numpy(chans).cuda())
    G = cfg.group
    for k in (100, 400):
        runs = {}
        for mode in ("1", "rescore", "0"):
            monkeypatch.setenv("TSD_TOPK_FILTER", mode)
            gidx, gcnt = tsd.topk_select_label(cache, index, queries, k)
            torch.cuda.synchronize()
            gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
            for t in range(len(w.kv_len)):
                b, L = int(w.token_seq[t]), int(w.kv_len[t])
                for h in range(cfg.num_q_heads):
                    K, _ = inp.kv(b, h // G)
                    s = oracle.label_scores(inp.q(t, h), K[:L], chans[h // G])
                    ok, why = oracle.topk_sets_agree(gidx[t, h], s, k, PT.TOPK_BAND)
                    assert ok, (mode, r, k, t, h, why)
                    assert int(gcnt[t, h]) == min(k, L)
            runs[mode] = gidx
        assert np.array_equal(runs["1"], runs["0"]), (r, k)
    assert tsd.read_device_status() == 0
