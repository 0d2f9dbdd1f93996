"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Small cases check every (token, head) list; they span several tiles, several
splits and ragged tails.  Full-size cases (the shapes of the workloads the
benchmark times) check a sample: every list of one sequence plus seeded
random lists.  Index lists fed to the GPU's sparse decode come from the
generator or from the oracle, never from the GPU.
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


def torch():
    import torch as _t
    return _t


def setup(w: W.HostWorkload, q_f32: bool = False):
    T = torch()
    dw = W.to_device(w, "cuda")
    contiguous = w.cfg.layout == "contiguous"
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=w.cfg.max_seq_len,
                        page_table=None if contiguous else dw.page_table)
    q = dw.q.float() if q_f32 else dw.q
    multi = w.cfg.tokens_per_seq > 1
    queries = tsd.Queries(q, q_indptr=dw.q_indptr if multi else None,
                          max_tokens_per_seq=w.cfg.tokens_per_seq, causal=w.cfg.causal, sm_scale=SM_SCALE)
    return dw, cache, queries


def all_pairs(w):
    return [(t, h) for t in range(len(w.kv_len)) for h in range(w.cfg.num_q_heads)]


def oracle_lists(inp: PT.OracleInputs, w, k_max, k_per_token, pairs):
    idx = np.full((len(w.kv_len), w.cfg.num_q_heads, k_max), -1, dtype=np.int32)
    for t, h in pairs:
        sel = inp.topk(t, h, int(k_per_token[t]))
        idx[t, h, :sel.size] = sel
    return idx


def fill_unsampled(idx, w, k_max):
    """Lists the oracle did not make get generator-made uniform lists."""
    uni = W.uniform_indices(w, k_max, seed_purpose=77)
    empty = (idx[:, :, 0] == -1)
    idx[empty] = uni[empty]
    return idx


def run_sparse(cache, queries, idx_np, out_f32):
    T = torch()
    idx = T.from_numpy(idx_np).cuda()
    out, lse = tsd.sparse_decode(cache, queries, idx, out_dtype=T.float32 if out_f32 else T.bfloat16)
    T.cuda.synchronize()
    return PT.bf16_to_np(out), lse.cpu().numpy()


# ---------------------------------------------------------------------------
def test_generator_device_matches_host():
    T = torch()
    for cfg, lens in ((W.CONFIGS["tiny"], None), (SMALL, SMALL_LENS)):
        w = W.make_workload(cfg, seed=3, seq_lens=lens)
        dw = W.to_device(w, "cuda")
        kflat = dw.k.view(T.int16).view(-1, 128)
        vflat = dw.v.view(T.int16).view(-1, 128)
        rng = np.random.default_rng(0)
        for _ in range(12):
            b = int(rng.integers(cfg.batch))
            g = int(rng.integers(cfg.num_kv_heads))
            toks = np.unique(rng.integers(0, int(w.seq_lens[b]), size=20))
            if cfg.planted:
                toks = np.unique(np.concatenate([toks, w.planted_k[(b, g)][0][:3], [0]]))
            rows = [w.physical_row(b, g, int(i)) for i in toks]
            rk = kflat[rows].cpu().numpy().view(np.uint16)
            rv = vflat[rows].cpu().numpy().view(np.uint16)
            assert np.array_equal(rk, w.logical_kv_bits(b, g, "k", toks))
            assert np.array_equal(rv, w.logical_kv_bits(b, g, "v", toks))


def test_tiny_config_full():
    T = torch()
    cfg = W.CONFIGS["tiny"]
    w = W.make_workload(cfg, seed=0)
    dw, cache, queries = setup(w)
    inp = PT.OracleInputs(w)
    kpt = w.k_per_token()
    idx, cnt = tsd.topk_select(cache, queries, 82)
    T.cuda.synchronize()
    stats = PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), kpt, all_pairs(w))
    assert stats["lists"] == 8
    # sparse decode on the oracle's lists, fp32 output (as the configuration asks)
    oidx = oracle_lists(inp, w, 82, kpt, all_pairs(w))
    out, lse = run_sparse(cache, queries, oidx, out_f32=True)
    PT.check_decode(inp, oidx, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    # the GPU pipeline (GPU lists -> GPU decode) against the oracle pipeline
    out2, lse2 = tsd.sparse_decode(cache, queries, idx, out_dtype=T.float32)
    gidx = idx.cpu().numpy()
    same = [(t, h) for (t, h) in all_pairs(w) if np.array_equal(gidx[t, h], oidx[t, h])]
    assert len(same) >= 7
    PT.check_decode(inp, oidx, PT.bf16_to_np(out2), lse2.cpu().numpy(), same, SM_SCALE, out_is_bf16=False)
    # dense
    outd, lsed = tsd.dense_decode(cache, queries, out_dtype=T.float32)
    PT.check_decode(inp, None, PT.bf16_to_np(outd), lsed.cpu().numpy(), all_pairs(w), SM_SCALE,
                    out_is_bf16=False, dense=True)
    assert tsd.read_device_status() == 0


@pytest.fixture(scope="module")
def small():
    w = W.make_workload(SMALL, seed=1, seq_lens=SMALL_LENS)
    dw, cache, queries = setup(w)
    return w, dw, cache, queries, PT.OracleInputs(w)


def test_small_topk(small):
    T = torch()
    w, dw, cache, queries, inp = small
    for k in (1, 100, 400):     # 400 > kv_len of the 300-token sequence
        idx, cnt = tsd.topk_select(cache, queries, k)
        T.cuda.synchronize()
        PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), w.k_per_token(k), all_pairs(w))
    # per-token k
    kpt = np.array([5, 77, 1, 300, 2500, 0], dtype=np.int32)
    idx, cnt = tsd.topk_select(cache, queries, 320, k_per_token=T.from_numpy(kpt).cuda())
    T.cuda.synchronize()
    PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), np.minimum(kpt, 320), all_pairs(w))
    assert tsd.read_device_status() == 0


@pytest.mark.parametrize("out_f32", [False, True])
def test_small_sparse_oracle_lists(small, out_f32):
    w, dw, cache, queries, inp = small
    kpt = w.k_per_token(100)
    oidx = oracle_lists(inp, w, 100, kpt, all_pairs(w))
    out, lse = run_sparse(cache, queries, oidx, out_f32)
    PT.check_decode(inp, oidx, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=not out_f32)
    assert tsd.read_device_status() == 0


@pytest.mark.parametrize("maker", ["uniform", "zipf"])
def test_small_sparse_generated_lists(small, maker):
    w, dw, cache, queries, inp = small
    for k in (7, 250, 3000):
        idx = W.uniform_indices(w, k) if maker == "uniform" else W.zipf_page_run_indices(w, k)
        out, lse = run_sparse(cache, queries, idx, out_f32=True)
        PT.check_decode(inp, idx, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    assert tsd.read_device_status() == 0


def test_small_pipeline(small):
    T = torch()
    w, dw, cache, queries, inp = small
    idx, cnt = tsd.topk_select(cache, queries, 100)
    out, lse = tsd.sparse_decode(cache, queries, idx)
    T.cuda.synchronize()
    kpt = w.k_per_token(100)
    oidx = oracle_lists(inp, w, 100, kpt, all_pairs(w))
    gidx = idx.cpu().numpy()
    same = [p for p in all_pairs(w) if np.array_equal(gidx[p], oidx[p])]
    assert len(same) >= 0.95 * len(all_pairs(w))
    PT.check_decode(inp, oidx, PT.bf16_to_np(out), lse.cpu().numpy(), same, SM_SCALE, out_is_bf16=True)


@pytest.mark.parametrize("out_f32", [False, True])
def test_small_dense(small, out_f32):
    T = torch()
    w, dw, cache, queries, inp = small
    out, lse = tsd.dense_decode(cache, queries, out_dtype=T.float32 if out_f32 else T.bfloat16)
    T.cuda.synchronize()
    PT.check_decode(inp, None, PT.bf16_to_np(out), lse.cpu().numpy(), all_pairs(w), SM_SCALE,
                    out_is_bf16=not out_f32, dense=True)


def test_sparse_with_every_token_equals_dense(small):
    w, dw, cache, queries, inp = small
    kmax = int(w.kv_len.max())
    idx = np.full((len(w.kv_len), w.cfg.num_q_heads, kmax), -1, dtype=np.int32)
    for t in range(len(w.kv_len)):
        idx[t, :, :w.kv_len[t]] = np.arange(w.kv_len[t])
    out, lse = run_sparse(cache, queries, idx, out_f32=True)
    PT.check_decode(inp, None, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False, dense=True)


def test_q_fp32_matches(small):
    T = torch()
    w, dw, cache, _, inp = small
    queries = tsd.Queries(dw.q.float(), q_indptr=dw.q_indptr, max_tokens_per_seq=2, causal=True, sm_scale=SM_SCALE)
    oidx = oracle_lists(inp, w, 100, w.k_per_token(100), all_pairs(w))
    out, lse = run_sparse(cache, queries, oidx, out_f32=True)
    PT.check_decode(inp, oidx, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    idx, cnt = tsd.topk_select(cache, queries, 100)
    T.cuda.synchronize()
    PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), w.k_per_token(100), all_pairs(w))


def test_edge_lists(small):
    """Duplicates (each occurrence a term), empty lists, -1 padding, k_max = 1."""
    T = torch()
    w, dw, cache, queries, inp = small
    Tn, Hq = len(w.kv_len), w.cfg.num_q_heads
    rng = np.random.default_rng(5)
    idx = np.full((Tn, Hq, 40), -1, dtype=np.int32)
    for t in range(Tn):
        L = int(w.kv_len[t])
        for h in range(Hq):
            kind = (t + h) % 4
            if kind == 0:      # duplicates
                base = np.sort(rng.integers(0, L, size=20))
                idx[t, h, :40] = np.sort(np.concatenate([base, base]))
            elif kind == 1:    # empty
                pass
            elif kind == 2:    # a single entry
                idx[t, h, 0] = int(rng.integers(0, L))
            else:              # last token only, twice
                idx[t, h, :2] = L - 1
    out, lse = run_sparse(cache, queries, idx, out_f32=True)
    PT.check_decode(inp, idx, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    assert tsd.read_device_status() == 0
    one = np.full((Tn, Hq, 1), -1, dtype=np.int32)
    for t in range(Tn):
        one[t, :, 0] = np.arange(Hq) % int(w.kv_len[t])
    out, lse = run_sparse(cache, queries, one, out_f32=True)
    PT.check_decode(inp, one, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)


def test_bad_entries_are_flagged_and_skipped(small):
    w, dw, cache, queries, inp = small
    Tn, Hq = len(w.kv_len), w.cfg.num_q_heads
    good = W.uniform_indices(w, 30)
    bad = good.copy()
    bad[0, 0, 29] = int(w.kv_len[0]) + 5          # beyond kv_len (still ascending)
    bad[1, 3, 29] = 2_000_000_000
    out, lse = run_sparse(cache, queries, bad, out_f32=True)
    flags = tsd.read_device_status()
    assert flags & tsd.DEV_BAD_INDEX
    expect = good.copy()
    expect[0, 0, 29] = -1
    expect[1, 3, 29] = -1
    PT.check_decode(inp, expect, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    # a descending list raises the ordering flag (its result is unspecified)
    uns = good.copy()
    uns[2, 1, :30] = uns[2, 1, :30][::-1]
    run_sparse(cache, queries, uns, out_f32=True)
    assert tsd.read_device_status() & tsd.DEV_UNSORTED


@pytest.mark.parametrize("page_size", [1, 8, 64])
def test_page_sizes(page_size):
    T = torch()
    cfg = W.DecodeConfig(name="pages", batch=2, num_q_heads=4, num_kv_heads=1, seq_len=3000, page_size=page_size,
                         ks=(64,), causal=True)
    w = W.make_workload(cfg, seed=2, seq_lens=[3000, 1234])
    dw, cache, queries = setup(w)
    inp = PT.OracleInputs(w)
    idx, cnt = tsd.topk_select(cache, queries, 64)
    T.cuda.synchronize()
    PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), w.k_per_token(64), all_pairs(w))
    lists = W.zipf_page_run_indices(w, 200)
    out, lse = run_sparse(cache, queries, lists, out_f32=True)
    PT.check_decode(inp, lists, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    outd, lsed = tsd.dense_decode(cache, queries, out_dtype=T.float32)
    T.cuda.synchronize()
    PT.check_decode(inp, None, PT.bf16_to_np(outd), lsed.cpu().numpy(), all_pairs(w), SM_SCALE,
                    out_is_bf16=False, dense=True)


@pytest.mark.parametrize("out_f32,with_lse", [(False, True), (True, True), (False, False)])
def test_host_buffers_match_the_device_path(small, out_f32, with_lse):
    """sparse_decode on pinned host q, lists, out and lse (one tsd_sparse_decode_host call:
    copies in, decode, copies back) gives exactly the device path's result, and the oracle's."""
    T = torch()
    w, dw, cache, queries, inp = small
    lists = W.uniform_indices(w, 250)
    odt = T.float32 if out_f32 else T.bfloat16
    out_d, lse_d = tsd.sparse_decode(cache, queries, T.from_numpy(lists).cuda(), out_dtype=odt)
    qh = tsd.Queries(dw.q.cpu().pin_memory(), q_indptr=dw.q_indptr, max_tokens_per_seq=SMALL.tokens_per_seq,
                     causal=True, sm_scale=SM_SCALE)
    out_h = T.empty(tuple(out_d.shape), dtype=odt).pin_memory()
    lse_h = T.empty(tuple(lse_d.shape), dtype=T.float32).pin_memory() if with_lse else None
    o, l = tsd.sparse_decode(cache, qh, T.from_numpy(lists).pin_memory(), out=out_h, lse=lse_h)
    T.cuda.synchronize()
    assert o.data_ptr() == out_h.data_ptr()
    assert T.equal(out_h, out_d.cpu())
    if with_lse:
        assert T.equal(lse_h, lse_d.cpu())
    else:
        assert l is None
    PT.check_decode(inp, lists, PT.bf16_to_np(out_h), lse_d.cpu().numpy(), all_pairs(w), SM_SCALE,
                    out_is_bf16=not out_f32)
    assert tsd.read_device_status() == 0


def test_host_buffers_with_fp32_queries(small):
    """The host-buffer call stages an fp32 q (4 bytes per element) the same way: it matches the
    device path on the same fp32 queries exactly."""
    T = torch()
    w, dw, cache, queries, inp = small
    lists = W.zipf_page_run_indices(w, 180)
    qf = dw.q.float()
    qd = tsd.Queries(qf, q_indptr=dw.q_indptr, max_tokens_per_seq=SMALL.tokens_per_seq, causal=True,
                     sm_scale=SM_SCALE)
    out_d, lse_d = tsd.sparse_decode(cache, qd, T.from_numpy(lists).cuda(), out_dtype=T.float32)
    qh = tsd.Queries(qf.cpu().pin_memory(), q_indptr=dw.q_indptr, max_tokens_per_seq=SMALL.tokens_per_seq,
                     causal=True, sm_scale=SM_SCALE)
    out_h = T.empty(tuple(out_d.shape), dtype=T.float32).pin_memory()
    lse_h = T.empty(tuple(lse_d.shape), dtype=T.float32).pin_memory()
    tsd.sparse_decode(cache, qh, T.from_numpy(lists).pin_memory(), out=out_h, lse=lse_h)
    T.cuda.synchronize()
    assert T.equal(out_h, out_d.cpu()) and T.equal(lse_h, lse_d.cpu())
    assert tsd.read_device_status() == 0


def test_ctas_spanning_two_sequences():
    """A shape whose tasks per sequence (kv heads x lists x chunks = 1 x 2 x 19) are not a
    multiple of a sparse-decode CTA's 4 warps: some CTAs hold the end of one sequence and the
    start of the next.  Those look pages up in global memory, the others in the page-table row
    they cached in shared memory; every list must match the oracle either way."""
    T = torch()
    cfg = W.DecodeConfig(name="straddle", batch=5, num_q_heads=2, num_kv_heads=1, seq_len=4096, ks=(300,),
                         planted=True, causal=True)
    w = W.make_workload(cfg, seed=5, seq_lens=[3000, 700, 4096, 1500, 2222])
    dw, cache, queries = setup(w)
    inp = PT.OracleInputs(w)
    idx, cnt = tsd.topk_select(cache, queries, 300)
    T.cuda.synchronize()
    PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), w.k_per_token(300), all_pairs(w))
    lists = oracle_lists(inp, w, 300, w.k_per_token(300), all_pairs(w))
    out, lse = run_sparse(cache, queries, lists, out_f32=True)
    PT.check_decode(inp, lists, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=False)
    for maker in (W.uniform_indices, W.zipf_page_run_indices):
        lists = maker(w, 300)
        out, lse = run_sparse(cache, queries, lists, out_f32=False)
        PT.check_decode(inp, lists, out, lse, all_pairs(w), SM_SCALE, out_is_bf16=True)
    assert tsd.read_device_status() == 0


def test_deterministic(small):
    T = torch()
    w, dw, cache, queries, inp = small
    a_idx, _ = tsd.topk_select(cache, queries, 100)
    a_idx = a_idx.clone()
    b_idx, _ = tsd.topk_select(cache, queries, 100)
    assert T.equal(a_idx, b_idx)
    o1, l1 = tsd.sparse_decode(cache, queries, a_idx)
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = tsd.sparse_decode(cache, queries, a_idx)
    assert T.equal(o1, o2) and T.equal(l1, l2)
    d1, _ = tsd.dense_decode(cache, queries)
    d1 = d1.clone()
    d2, _ = tsd.dense_decode(cache, queries)
    assert T.equal(d1, d2)


# ---------------------------------------------------------------------------
# Full-size workloads (sampled lists)
# ---------------------------------------------------------------------------
def _full_topk_and_decode(cfg_name, ks, n_random=6, full_seqs=(0,), check_dense=True):
    T = torch()
    cfg = W.CONFIGS[cfg_name]
    w = W.make_workload(cfg, seed=0)
    dw, cache, queries = setup(w)
    inp = PT.OracleInputs(w)
    pairs = PT.sample_pairs(w, n_random, full_seqs=full_seqs, seed=1)
    for k in ks:
        kpt = w.k_per_token(k)
        k_max = int(kpt.max())
        idx, cnt = tsd.topk_select(cache, queries, k_max,
                                   k_per_token=None if k is not None else T.from_numpy(kpt).cuda())
        T.cuda.synchronize()
        PT.check_topk(inp, idx.cpu().numpy(), cnt.cpu().numpy(), kpt, pairs)
        # the decode on lists made by the oracle for the sampled pairs
        oidx = fill_unsampled(oracle_lists(inp, w, k_max, kpt, pairs), w, k_max)
        out, lse = run_sparse(cache, queries, oidx, out_f32=False)
        PT.check_decode(inp, oidx, out, lse, pairs, SM_SCALE, out_is_bf16=True)
        # the GPU pipeline where the sets agree exactly
        out2, lse2 = tsd.sparse_decode(cache, queries, idx)
        gidx = idx.cpu().numpy()
        same = [p for p in pairs if np.array_equal(gidx[p], oidx[p])]
        assert len(same) >= 0.9 * len(pairs)
        PT.check_decode(inp, oidx, PT.bf16_to_np(out2), lse2.cpu().numpy(), same, SM_SCALE, out_is_bf16=True)
    if check_dense:
        outd, lsed = tsd.dense_decode(cache, queries)
        T.cuda.synchronize()
        PT.check_decode(inp, None, PT.bf16_to_np(outd), lsed.cpu().numpy(), pairs, SM_SCALE,
                        out_is_bf16=True, dense=True)
    assert tsd.read_device_status() == 0


def test_full_llama3_8b():
    _full_topk_and_decode("llama3_8b", ks=(655,))


def test_full_qwen25_72b():
    _full_topk_and_decode("qwen25_72b", ks=(2621, 13107, 1311), n_random=4)


def test_full_ragged():
    _full_topk_and_decode("ragged", ks=(None,), n_random=6)


def test_full_sweep():
    T = torch()
    cfg = W.CONFIGS["sweep"]
    w = W.make_workload(cfg, seed=0)
    dw, cache, queries = setup(w)
    inp = PT.OracleInputs(w)
    pairs = PT.sample_pairs(w, 4, full_seqs=(0,), seed=2)
    for k in cfg.ks:
        for maker in (W.uniform_indices, W.zipf_page_run_indices):
            idx = maker(w, k)
            out, lse = run_sparse(cache, queries, idx, out_f32=False)
            PT.check_decode(inp, idx, out, lse, pairs, SM_SCALE, out_is_bf16=True)
    outd, lsed = tsd.dense_decode(cache, queries)
    T.cuda.synchronize()
    PT.check_decode(inp, None, PT.bf16_to_np(outd), lsed.cpu().numpy(), pairs, SM_SCALE, out_is_bf16=True,
                    dense=True)
    assert tsd.read_device_status() == 0
