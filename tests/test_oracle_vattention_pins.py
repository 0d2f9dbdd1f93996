"""Pins of the stochastic-selection oracle (vAttention-style), and mutants they must catch.

Facts used:
* Floyd's algorithm: hand traces, and exact uniformity -- enumerating every combination of
  the random draws, each m-subset of [0, n) comes out equally often (C(n, m) divides the
  number of draw combinations n! / (n - m)!);
* the estimator is unbiased: averaged over every equally likely sample, the weighted sum over
  the sampled tokens equals the exact sum over the rest (exact enumeration, small n);
* sampling all of the rest reproduces dense attention (a separately pinned oracle function);
* the weights of a list add up to its length; V = 1 gives 1; a hand example of weighting.
"""

import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import vattention as VA


def check_floyd(floyd_sample):
    assert floyd_sample(5, 3, [2, 2, 4]).tolist() == [2, 3, 4]
    assert floyd_sample(5, 3, [0, 1, 0]).tolist() == [0, 1, 4]
    assert floyd_sample(4, 4, [9, 9, 9, 9]).tolist() == [0, 1, 2, 3]
    for n, m in ((5, 2), (6, 3), (4, 1)):
        counts = {}
        ranges = [range(j + 1) for j in range(n - m, n)]
        for draws in itertools.product(*ranges):
            key = tuple(floyd_sample(n, m, list(draws)).tolist())
            assert len(key) == m and len(set(key)) == m and all(0 <= x < n for x in key)
            counts[key] = counts.get(key, 0) + 1
        assert len(counts) == math.comb(n, m)
        assert len(set(counts.values())) == 1, (n, m, counts)


def check_unbiased(stochastic_select):
    rng = np.random.default_rng(3)
    s = rng.standard_normal(8)
    k, m = 2, 3
    top = oracle.exact_topk(s, k)
    rest = np.setdiff1d(np.arange(8), top)
    exact = np.exp(s[rest]).sum()
    n = rest.size
    total, count = 0.0, 0
    ranges = [range(j + 1) for j in range(n - m, n)]
    for draws in itertools.product(*ranges):   # every draw combination is equally likely
        idx, lw = stochastic_select(s, k, m, list(draws))
        samp = np.setdiff1d(idx, top)
        w = np.exp(lw[np.isin(idx, samp)])
        total += float((w * np.exp(s[samp])).sum())
        count += 1
    assert abs(total / count - exact) <= 1e-12 * exact


def check_weights_and_limits(stochastic_select, weighted_attention):
    rng = np.random.default_rng(4)
    L, D = 40, 16
    q, K, V = rng.standard_normal(D), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    s = K @ q
    u = rng.integers(0, 2**32, size=64, dtype=np.uint64)
    idx, lw = stochastic_select(s, 5, 7, u)
    assert np.all(np.diff(idx) > 0) and idx.size == 12
    assert abs(np.exp(lw).sum() - L) < 1e-9                      # weights add up to L
    assert set(oracle.exact_topk(s, 5).tolist()) <= set(idx.tolist())
    ones = np.ones((L, D))
    o1, _ = weighted_attention(q, K, ones, idx, lw, 0.25)
    assert np.allclose(o1, 1.0, rtol=0, atol=1e-12)
    idx_all, lw_all = stochastic_select(s, 5, L, u)              # the whole rest is sampled
    assert idx_all.tolist() == list(range(L)) and np.allclose(lw_all, 0.0)
    o, lse = weighted_attention(q, K, V, idx_all, lw_all, 0.25)
    od, lsed = oracle.dense_attention(q, K, V, 0.25)
    assert np.allclose(o, od, rtol=0, atol=1e-12) and abs(lse - lsed) < 1e-12


def check_weighted_hand(weighted_attention):
    q, K = np.array([1.0]), np.array([[0.0], [0.0]])
    V = np.array([[1.0], [3.0]])
    out, lse = weighted_attention(q, K, V, np.array([0, 1]), np.array([0.0, math.log(3.0)]), 1.0)
    assert abs(out[0] - 2.5) < 1e-12 and abs(lse - math.log(4.0)) < 1e-12


def test_vattention_pins_hold():
    check_floyd(oracle.floyd_sample)
    check_unbiased(oracle.stochastic_select)
    check_weights_and_limits(oracle.stochastic_select, oracle.weighted_attention)
    check_weighted_hand(oracle.weighted_attention)


def _floyd_collision_keeps_t(n, m, u):
    m = max(0, min(int(m), int(n)))
    chosen = []
    for step, j in enumerate(range(n - m, n)):
        t = int(np.uint64(u[step]) % np.uint64(j + 1))
        if t not in chosen:
            chosen.append(t)
    return np.array(sorted(chosen), dtype=np.int64)


def _select_inverted_weight(s, k, m, u):
    idx, lw = VA.stochastic_select(s, k, m, u)
    return idx, -lw


def _select_weights_everything(s, k, m, u):
    idx, lw = VA.stochastic_select(s, k, m, u)
    return idx, np.full_like(lw, lw.max())


def _select_from_all_tokens(s, k, m, u):
    s = np.asarray(s, dtype=np.float64)
    top = oracle.exact_topk(s, k)
    L = s.shape[0]
    samp = VA.floyd_sample(L, m, u)
    idx = np.union1d(top, samp)
    lw = np.where(np.isin(idx, top), 0.0, math.log((L - top.size) / max(1, m)))
    return idx, lw


def _weighted_ignores_weights(q, K, V, idx, logw, sm):
    return VA.weighted_attention(q, K, V, idx, np.zeros_like(np.asarray(logw, dtype=float)), sm)


@pytest.mark.parametrize("name,check", [
    ("floyd keeps t on a collision", lambda: check_floyd(_floyd_collision_keeps_t)),
    ("inverted sample weight", lambda: check_unbiased(_select_inverted_weight)),
    ("top-k weighted like samples", lambda: check_weights_and_limits(_select_weights_everything,
                                                                      oracle.weighted_attention)),
    ("sampling from every token", lambda: check_unbiased(_select_from_all_tokens)),
    ("weights ignored", lambda: check_weighted_hand(_weighted_ignores_weights)),
])
def test_vattention_mutants_are_caught(name, check):
    with pytest.raises(AssertionError):
        check()
