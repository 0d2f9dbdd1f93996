"""The seeded input generator: published Philox answers, distributions, structure."""

import math

import numpy as np
import pytest

from top_sparse_decode_topk_b200 import workload as W


def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 published with the Random123 library.
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for ctr, key, want in cases:
        got = W.philox4x32_10(*[np.array([c], dtype=np.uint64) for c in ctr], *key)
        assert tuple(int(x[0]) for x in got) == want


def test_normal_table_symmetric_and_standard():
    t = W.bf16_bits_to_f64(W.normal_table())
    assert np.array_equal(t, -t[::-1])             # exact antisymmetry -> mean 0
    assert abs(t.mean()) < 1e-12
    assert abs(t.var() - 1.0) < 2e-3
    assert np.all(np.diff(t) >= 0)


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.140625], dtype=np.float32)
    got = W.bf16_bits_to_f32(W.f32_to_bf16_bits(x))
    assert got.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 3.140625]


def test_base_values_reproducible_and_independent():
    a = W.kv_base_bits(0, W.TENSOR_K, 1, 2, np.arange(64))
    b = W.kv_base_bits(0, W.TENSOR_K, 1, 2, np.arange(64))
    c = W.kv_base_bits(0, W.TENSOR_V, 1, 2, np.arange(64))
    d = W.kv_base_bits(1, W.TENSOR_K, 1, 2, np.arange(64))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # a sub-range regenerates the same rows
    assert np.array_equal(W.kv_base_bits(0, W.TENSOR_K, 1, 2, np.arange(10, 20)), a[10:20])
    x = W.bf16_bits_to_f64(W.kv_base_bits(3, W.TENSOR_V, 0, 0, np.arange(4096)))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_k_rounding_matches_configs():
    assert W.k_for_sparsity(4096, 50) == 82
    assert W.k_for_sparsity(32768, 50) == 655
    assert [W.k_for_sparsity(131072, x) for x in (10, 50, 100)] == [13107, 2621, 1311]
    assert W.CONFIGS["sweep"].ks == (65536, 16384, 6554, 2621, 1311, 655, 328)


def test_tiny_workload_shapes():
    w = W.make_workload(W.CONFIGS["tiny"], seed=0)
    assert w.q_bits.shape == (1, 8, 128)
    assert w.page_table.shape == (1, 1) and w.page_size == 4096
    assert w.kv_len.tolist() == [4096]
    assert w.k_per_token().tolist() == [82]


def test_paged_table_is_a_permutation():
    w = W.make_workload(W.CONFIGS["llama3_8b"], seed=0)
    used = w.page_table[w.page_table >= 0]
    assert used.size == w.num_pages == 8 * 2048
    assert np.array_equal(np.sort(used), np.arange(w.num_pages))
    # physical order is shuffled
    assert not np.array_equal(w.page_table[0, :16], np.arange(16))


def test_planted_structure_cosines():
    w = W.make_workload(W.CONFIGS["llama3_8b"], seed=0)
    q = W.bf16_bits_to_f64(w.q_bits)
    G = w.cfg.group
    b, g = 3, 5
    pos, bits = w.planted_k[(b, g)]
    rows = W.bf16_bits_to_f64(bits)
    assert pos[-128:].tolist() == list(range(32768 - 128, 32768))
    assert pos[64] == 0
    for j in range(64):
        h = g * G + j % G
        cos = rows[j] @ q[b, h] / (np.linalg.norm(rows[j]) * np.linalg.norm(q[b, h]))
        assert abs(cos - 0.5) < 0.01
        assert abs(np.linalg.norm(rows[j]) - math.sqrt(128)) < 0.1
    m = np.mean([q[b, g * G + j] for j in range(G)], axis=0)
    m /= np.linalg.norm(m)
    assert abs(rows[64] @ m / np.linalg.norm(rows[64]) - 0.9) < 0.01
    for r in rows[65:]:
        assert abs(r @ m / np.linalg.norm(r) - 0.5) < 0.01
    # logical rows carry the planted values
    got = w.logical_kv_bits(b, g, "k", pos[:3])
    assert np.array_equal(got, bits[:3])


def test_ragged_lengths_and_causal_kv_len():
    w = W.make_workload(W.CONFIGS["ragged"], seed=0)
    assert w.seq_lens.min() >= 8192 and w.seq_lens.max() <= 131072
    assert len(set(w.seq_lens.tolist())) > 20
    for b in range(32):
        L = int(w.seq_lens[b])
        assert w.kv_len[4 * b:4 * b + 4].tolist() == [L - 3, L - 2, L - 1, L]
    k = w.k_per_token()
    assert np.array_equal(k, np.ceil(0.02 * w.kv_len - 1e-12).astype(np.int32))


@pytest.mark.parametrize("maker", ["uniform", "zipf"])
def test_supplied_index_lists(maker):
    cfg = W.DecodeConfig(name="sweep", batch=2, num_q_heads=4, num_kv_heads=2, seq_len=4096)
    w = W.make_workload(cfg, seed=0)
    k = 300
    idx = W.uniform_indices(w, k) if maker == "uniform" else W.zipf_page_run_indices(w, k)
    assert idx.shape == (2, 4, k)
    for t in range(2):
        for h in range(4):
            row = idx[t, h]
            assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < 4096
    if maker == "zipf":
        # clustered: most selected tokens come in whole 16-token pages
        pages = idx[0, 0] // 16
        _, counts = np.unique(pages, return_counts=True)
        assert (counts == 16).sum() >= (k // 16) - 1
