"""The persistent sparse-decode kernel on the cases its chunking makes special (needs a B200).

The library runs the persistent form when the one-task-per-warp plan would need more than
one wave of CTAs (the ragged workload); TSD_SPARSE_KERNEL=stream forces it and
TSD_SPARSE_CHUNK sets its entries per task, so that small lists span many chunks here.  The
cases: lists whose length is exactly a multiple of the chunk (the list's end is only seen from
the next chunk's first entry), empty lists over many chunks, single entries, lists one entry
short of or past a chunk boundary, repeated tokens, per-token k with multi-token decode, the
weighted form, and entries the kernel must flag and skip.  Every list is compared with the
float64 oracle on the same inputs.
"""

import math

import numpy as np
import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
CFG = W.DecodeConfig(name="stream_small", batch=5, num_q_heads=8, num_kv_heads=2, seq_len=5000, tokens_per_seq=3,
                     ks=(200,), planted=True, causal=True)
LENS = [5000, 700, 4096, 1500, 2222]


@pytest.fixture
def stream_form(monkeypatch):
    monkeypatch.setenv("TSD_SPARSE_KERNEL", "stream")
    monkeypatch.setenv("TSD_SPARSE_CHUNK", "64")


@pytest.fixture(scope="module")
def case():
    w = W.make_workload(CFG, seed=6, seq_lens=LENS)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=CFG.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr, max_tokens_per_seq=CFG.tokens_per_seq, causal=True,
                          sm_scale=SM_SCALE)
    return w, cache, queries, PT.OracleInputs(w)


def _pairs(w):
    return [(t, h) for t in range(len(w.kv_len)) for h in range(w.cfg.num_q_heads)]


def _edge_lists(w, k_max, seed=0):
    """Lists with lengths at and around multiples of the 64-entry chunk, empty lists, single
    entries and repeated tokens, all ascending and -1 padded."""
    rng = np.random.default_rng(seed)
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    idx = np.full((T, Hq, k_max), -1, dtype=np.int32)
    lengths = [0, 1, 63, 64, 65, 127, 128, 129, 192, k_max]
    for t in range(T):
        L = int(w.kv_len[t])
        for h in range(Hq):
            n = lengths[(t * Hq + h) % len(lengths)]
            if n == 0:
                continue
            if (t + h) % 5 == 0:   # repeated tokens: each occurrence is a term
                base = np.sort(rng.integers(0, L, size=(n + 1) // 2))
                sel = np.sort(np.concatenate([base, base]))[:n]
            else:
                sel = np.sort(rng.choice(L, size=min(n, L), replace=False))
            idx[t, h, :sel.size] = sel
    return idx


def _run(cache, queries, idx_np, f32=True, logw=None):
    import torch
    idx = torch.from_numpy(idx_np).cuda()
    lw = None if logw is None else torch.from_numpy(logw).cuda()
    out, lse = tsd.sparse_decode(cache, queries, idx, out_dtype=torch.float32 if f32 else torch.bfloat16, logw=lw)
    torch.cuda.synchronize()
    return PT.bf16_to_np(out), lse.cpu().numpy()


def test_chunk_boundaries_and_empty_lists(stream_form, case):
    w, cache, queries, inp = case
    idx = _edge_lists(w, 300)
    out, lse = _run(cache, queries, idx)
    assert tsd.read_device_status() == 0
    PT.check_decode(inp, idx, out, lse, _pairs(w), SM_SCALE, out_is_bf16=False)
    out2, lse2 = _run(cache, queries, idx)   # the counters were left zero: a second call agrees exactly
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_uniform_and_page_run_lists_bf16(stream_form, case):
    w, cache, queries, inp = case
    for maker in (W.uniform_indices, W.zipf_page_run_indices):
        idx = maker(w, 200)
        out, lse = _run(cache, queries, idx, f32=False)
        PT.check_decode(inp, idx, out, lse, _pairs(w), SM_SCALE, out_is_bf16=True)
    assert tsd.read_device_status() == 0


def test_oracle_top_k_with_per_token_k(stream_form, case):
    """Lists from the oracle's exact top-k with k = ceil(0.02 kv_len) + 60, so that the lists of
    one sequence differ in length and some end inside the last chunk."""
    w, cache, queries, inp = case
    kpt = np.array([int(math.ceil(0.02 * L)) + 60 for L in w.kv_len], dtype=np.int32)
    k_max = int(kpt.max())
    idx = np.full((len(w.kv_len), CFG.num_q_heads, k_max), -1, dtype=np.int32)
    for t, h in _pairs(w):
        sel = inp.topk(t, h, int(kpt[t]))
        idx[t, h, :sel.size] = sel
    out, lse = _run(cache, queries, idx)
    PT.check_decode(inp, idx, out, lse, _pairs(w), SM_SCALE, out_is_bf16=False)
    assert tsd.read_device_status() == 0


def test_weighted_form(stream_form, case):
    """Entry weights exp(logw) through the persistent kernel: equal to the oracle's softmax over
    the list with ln w added to each scaled score (the vAttention estimator's form)."""
    import oracle
    w, cache, queries, inp = case
    idx = W.uniform_indices(w, 150)
    rng = np.random.default_rng(3)
    logw = np.where(idx >= 0, rng.uniform(-1.0, 2.0, size=idx.shape), 0.0).astype(np.float32)
    out, lse = _run(cache, queries, idx, logw=logw)
    for t, h in _pairs(w):
        b = inp.seq_of(t)
        K, V = inp.kv(b, h // CFG.group)
        L = int(w.kv_len[t])
        n = int((idx[t, h] >= 0).sum())
        o_ref, l_ref = oracle.weighted_attention(inp.q(t, h), K[:L], V[:L], idx[t, h, :n],
                                                 logw[t, h, :n].astype(np.float64), SM_SCALE)
        ok, why = oracle.output_within(out[t, h], o_ref, PT.F32_MAX_ABS, math.inf, False)
        assert ok, f"(t={t}, h={h}): {why}"
        assert abs(float(lse[t, h]) - l_ref) <= PT.LSE_ABS + 1e-5 * abs(l_ref)
    assert tsd.read_device_status() == 0


def test_bad_entries_flagged_and_skipped(stream_form, case):
    w, cache, queries, inp = case
    good = W.uniform_indices(w, 130)
    bad = good.copy()
    bad[0, 0, 129] = int(w.kv_len[0]) + 5     # past kv_len, in the third chunk
    bad[4, 3, 70] = 2_000_000_000             # far past, in the second chunk (the list stays ascending)
    bad[4, 3, 71:130] = -1
    out, lse = _run(cache, queries, bad)
    assert tsd.read_device_status() & tsd.DEV_BAD_INDEX
    expect = good.copy()
    expect[0, 0, 129] = -1
    expect[4, 3, 70:] = -1
    PT.check_decode(inp, expect, out, lse, _pairs(w), SM_SCALE, out_is_bf16=False)
