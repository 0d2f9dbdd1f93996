"""Checks that pin the oracle to facts outside itself.

Each check takes the functions under test as arguments so that the same
check can be run against deliberately broken copies (see test_oracle_pins.py,
which asserts that every planted mistake is caught by at least one check).
Sources of the facts:
* hand-derived closed forms in tests/golden/closed_forms.json;
* brute force over every k-subset of tiny contexts (top-k);
* k = N reproducing dense attention computed by a library routine
  (torch scaled_dot_product_attention in float64 on the CPU);
* k = 1 returning the V row of the arg-max; V = 1 giving 1; list-order
  invariance; the two-token logistic closed form; split-and-merge invariance.
"""

from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def check_golden_attention(sparse_attention):
    for case in _golden()["attention"]:
        out, lse = sparse_attention(np.array(case["q"]), np.array(case["K"]), np.array(case["V"]),
                                    np.array(case["idx"]), case["sm_scale"])
        assert np.allclose(out, case["out"], rtol=0, atol=1e-12), (case["name"], out)
        want = float(case["lse"]) if case["lse"] != "-inf" else -math.inf
        if math.isinf(want):
            assert math.isinf(lse) and lse < 0, (case["name"], lse)
        else:
            assert abs(lse - want) < 1e-12, (case["name"], lse, want)


def check_golden_topk(exact_topk):
    for case in _golden()["topk"]:
        got = exact_topk(np.array(case["scores"], dtype=np.float64), case["k"])
        assert list(map(int, got)) == case["selected"], (case["name"], got)


def brute_force_topk(scores, k):
    """Pure-Python reference: among the k-subsets in which every kept score is
    >= every dropped score, the lexicographically smallest (= ties to lower index)."""
    L = len(scores)
    n = min(k, L)
    best = None
    for sub in itertools.combinations(range(L), n):
        kept = set(sub)
        lo = min((scores[i] for i in sub), default=math.inf)
        hi = max((scores[i] for i in range(L) if i not in kept), default=-math.inf)
        if lo >= hi:
            if best is None or sub < best:
                best = sub
    return list(best)


def check_topk_brute_force(exact_topk, seed=0, trials=300):
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        L = int(rng.integers(1, 10))
        k = int(rng.integers(1, L + 2))
        if rng.random() < 0.5:
            s = rng.integers(-2, 3, size=L).astype(np.float64)  # many ties
        else:
            s = rng.standard_normal(L)
        got = list(map(int, exact_topk(s, k)))
        assert got == brute_force_topk(list(s), k), (s, k, got)


def check_topk_invariants(exact_topk, seed=1, trials=200):
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        L = int(rng.integers(1, 400))
        k = int(rng.integers(1, 500))
        s = rng.standard_normal(L) * rng.uniform(0.1, 100)
        got = np.asarray(exact_topk(s, k))
        n = min(k, L)
        assert got.shape == (n,)
        assert np.all(np.diff(got) > 0) and (n == 0 or (got[0] >= 0 and got[-1] < L))
        if 0 < n < L:
            rest = np.setdiff1d(np.arange(L), got)
            assert s[got].min() >= s[rest].max()


def check_planted_needles(exact_topk, attention_scores, seed=2):
    """Keys exactly aligned with the query and of large norm are always kept."""
    rng = np.random.default_rng(seed)
    D, L = 128, 2048
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, D))
    needles = rng.choice(L, size=20, replace=False)
    K[needles] = 8.0 * q / np.linalg.norm(q) * math.sqrt(D)
    got = exact_topk(attention_scores(q, K), 41)
    assert set(needles.tolist()) <= set(map(int, got))


def _sdpa(q, K, V, scale):
    import torch
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64)).view(1, 1, 1, -1)
    kt = torch.from_numpy(np.asarray(K, dtype=np.float64)).view(1, 1, K.shape[0], -1)
    vt = torch.from_numpy(np.asarray(V, dtype=np.float64)).view(1, 1, V.shape[0], -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o.view(-1).numpy()


def check_dense_matches_library(sparse_attention, dense_attention, seed=3):
    rng = np.random.default_rng(seed)
    for L, D in ((1, 8), (7, 16), (300, 128), (1000, 64)):
        q = rng.standard_normal(D) * 2.0
        K = rng.standard_normal((L, D))
        V = rng.standard_normal((L, D))
        scale = 1.0 / math.sqrt(D)
        ref = _sdpa(q, K, V, scale)
        o_dense, lse_d = dense_attention(q, K, V, scale)
        o_full, lse_f = sparse_attention(q, K, V, np.arange(L), scale)
        assert np.allclose(o_dense, ref, atol=1e-12, rtol=1e-10)
        assert np.allclose(o_full, ref, atol=1e-12, rtol=1e-10)
        z = scale * (K @ q)
        lse_ref = float(np.log(np.sum(np.exp(z - z.max()))) + z.max())
        assert abs(lse_d - lse_ref) < 1e-10 and abs(lse_f - lse_ref) < 1e-10


def check_k1_argmax_row(sparse_attention, exact_topk, attention_scores, seed=4):
    rng = np.random.default_rng(seed)
    D, L = 128, 513
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, D))
    V = rng.standard_normal((L, D))
    s = attention_scores(q, K)
    idx = exact_topk(s, 1)
    assert int(idx[0]) == int(np.argmax(s))
    out, lse = sparse_attention(q, K, V, idx, 0.125)
    assert np.array_equal(out, V[int(np.argmax(s))])
    assert abs(lse - 0.125 * s.max()) < 1e-12


def check_v_ones(sparse_attention, seed=5):
    rng = np.random.default_rng(seed)
    D, L = 64, 400
    q = rng.standard_normal(D) * 3
    K = rng.standard_normal((L, D))
    V = np.ones((L, D))
    idx = np.sort(rng.choice(L, 37, replace=False))
    out, _ = sparse_attention(q, K, V, idx, 0.2)
    assert np.allclose(out, 1.0, atol=1e-14)


def check_permutation_invariance(sparse_attention, seed=6):
    rng = np.random.default_rng(seed)
    D, L = 32, 257
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, D))
    V = rng.standard_normal((L, D))
    idx = rng.choice(L, 50, replace=False)
    a, la = sparse_attention(q, K, V, np.sort(idx), 0.3)
    b, lb = sparse_attention(q, K, V, rng.permutation(idx), 0.3)
    assert np.allclose(a, b, atol=1e-13) and abs(la - lb) < 1e-12


def check_two_token_logistic(sparse_attention, seed=7):
    rng = np.random.default_rng(seed)
    for _ in range(50):
        D = int(rng.integers(1, 9))
        q = rng.standard_normal(D)
        K = rng.standard_normal((2, D))
        V = rng.standard_normal((2, D))
        scale = float(rng.uniform(0.05, 2))
        delta = scale * (K[0] @ q - K[1] @ q)
        sig = 1.0 / (1.0 + math.exp(-delta))
        out, lse = sparse_attention(q, K, V, np.array([0, 1]), scale)
        assert np.allclose(out, sig * V[0] + (1 - sig) * V[1], atol=1e-13)
        z0, z1 = scale * (K[0] @ q), scale * (K[1] @ q)
        assert abs(lse - math.log(math.exp(z0) + math.exp(z1))) < 1e-12


def check_split_merge(sparse_attention, seed=8):
    """Attention over a list equals the log-sum-exp merge of any partition of it."""
    rng = np.random.default_rng(seed)
    D, L = 128, 1000
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, D))
    V = rng.standard_normal((L, D))
    idx = rng.choice(L, 300, replace=False)
    whole, lse_whole = sparse_attention(q, K, V, idx, 0.09)
    cuts = np.sort(rng.choice(np.arange(1, 300), size=6, replace=False))
    parts = [sparse_attention(q, K, V, p, 0.09) for p in np.split(idx, cuts)]
    M = max(l for _, l in parts)
    wts = np.array([math.exp(l - M) for _, l in parts])
    merged = sum(w * o for w, (o, _) in zip(wts, parts)) / wts.sum()
    assert np.allclose(merged, whole, atol=1e-13)
    assert abs(M + math.log(wts.sum()) - lse_whole) < 1e-12


ALL_ATTENTION_CHECKS = (
    "golden_attention", "dense_matches_library", "k1_argmax_row", "v_ones",
    "permutation_invariance", "two_token_logistic", "split_merge")
ALL_TOPK_CHECKS = ("golden_topk", "topk_brute_force", "topk_invariants", "planted_needles", "k1_argmax_row")


def run_all(sparse_attention, dense_attention, exact_topk, attention_scores):
    """Run every check; returns the list of names that failed."""
    checks = {
        "golden_attention": lambda: check_golden_attention(sparse_attention),
        "golden_topk": lambda: check_golden_topk(exact_topk),
        "topk_brute_force": lambda: check_topk_brute_force(exact_topk, trials=120),
        "topk_invariants": lambda: check_topk_invariants(exact_topk, trials=60),
        "planted_needles": lambda: check_planted_needles(exact_topk, attention_scores),
        "dense_matches_library": lambda: check_dense_matches_library(sparse_attention, dense_attention),
        "k1_argmax_row": lambda: check_k1_argmax_row(sparse_attention, exact_topk, attention_scores),
        "v_ones": lambda: check_v_ones(sparse_attention),
        "permutation_invariance": lambda: check_permutation_invariance(sparse_attention),
        "two_token_logistic": lambda: check_two_token_logistic(sparse_attention),
        "split_merge": lambda: check_split_merge(sparse_attention),
    }
    failed = []
    for name, fn in checks.items():
        try:
            fn()
        except Exception:
            failed.append(name)
    return failed
