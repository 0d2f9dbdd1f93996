"""Top-k selection with exact ties, checked index for index (needs a B200).

Each (sequence, kv head) cache is built from a pool of only a few distinct key rows, so
every list's scores take a few values, each shared by thousands of tokens.  Identical rows
give bit-identical fp32 dots on the GPU, so the selection has to apply the tie rule of the
oracle (lower token index first, "Oracle Top-K" in section 2 of the pages' summary): the
result must equal the oracle's list exactly, not just within the rounding band.  With two
distinct rows a tie group holds about half of a 32768-token list, more candidates than the
selection gathers in one place, so the full three-round radix path runs; with five rows the
candidate path runs; with 200 rows the groups are small enough for the sampled-threshold
path, and the k-th score still falls inside a group of about 160 equal scores.
"""

import math

import numpy as np
import pytest

import oracle
import top_sparse_decode_topk_b200 as tsd

pytestmark = pytest.mark.gpu

SEQ_LENS = [32768, 20001]
HKV, HQ, D = 2, 4, 128


def _hash(i: np.ndarray, salt: int) -> np.ndarray:
    x = (i.astype(np.uint64) + np.uint64(salt)) * np.uint64(2654435761)
    return (x >> np.uint64(7)) & np.uint64(0xFFFFFFFF)


def _bf16_round(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32)


def _tied_cache(n_distinct: int, seed: int):
    rng = np.random.default_rng(seed)
    B, N = len(SEQ_LENS), max(SEQ_LENS)
    K = np.zeros((B, HKV, N, D), dtype=np.float32)
    for b in range(B):
        for g in range(HKV):
            pool = _bf16_round(rng.standard_normal((n_distinct, D)).astype(np.float32))
            ids = (_hash(np.arange(N), 97 * b + g) % np.uint64(n_distinct)).astype(np.int64)
            K[b, g] = pool[ids]
    q = _bf16_round(rng.standard_normal((B, HQ, D)).astype(np.float32))
    return K, q


@pytest.mark.parametrize("n_distinct", [2, 5, 200])
def test_topk_ties_go_to_lower_indices(n_distinct):
    import torch
    K, q = _tied_cache(n_distinct, seed=11 + n_distinct)
    B, N = K.shape[0], K.shape[2]
    kd = torch.from_numpy(K).to(torch.bfloat16).cuda()
    vd = torch.zeros_like(kd)
    lens = torch.tensor(SEQ_LENS, dtype=torch.int32).cuda()
    cache = tsd.KVCache(kd, vd, lens, max_seq_len=N, page_table=None)
    queries = tsd.Queries(torch.from_numpy(q).to(torch.bfloat16).cuda(), sm_scale=1.0 / math.sqrt(D))
    G = HQ // HKV
    for k in (1, 100, 1000, 9000, 20000, 32768):
        idx, cnt = tsd.topk_select(cache, queries, k)
        torch.cuda.synchronize()
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            L = SEQ_LENS[b]
            for h in range(HQ):
                s = oracle.attention_scores(q[b, h].astype(np.float64), K[b, h // G, :L].astype(np.float64))
                ref = oracle.exact_topk(s, k)
                n = ref.size
                assert cnt[b, h] == n, (n_distinct, k, b, h)
                assert np.array_equal(idx[b, h, :n], ref), (n_distinct, k, b, h)
                assert np.all(idx[b, h, n:] == -1), (n_distinct, k, b, h)
    assert tsd.read_device_status() == 0
