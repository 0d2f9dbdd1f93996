"""Pins of the approximate (label-channel) indexer's oracle, and mutants they must catch.

Facts used (none of them re-types the oracle's own formula):
* keeping every channel must reproduce the exact attention scores (a different oracle
  function, itself pinned by brute force and closed forms);
* with one channel c the score of token i is the product q_c K[i, c], checked against a
  hand-made example;
* the channel set, not its order, defines the score;
* the importance is a sum of |q_d K_{i,d}| over all (query, token) pairs: brute-force double
  loop on tiny inputs, and a hand example;
* the channel choice keeps the largest importances, ties to the lower channel index: hand
  examples, and brute force over every r-subset of a tiny channel count.
"""

import itertools

import numpy as np
import pytest

import oracle
from oracle import label as Lb


def check_all_channels_is_exact(label_scores):
    rng = np.random.default_rng(5)
    q, K = rng.standard_normal(128), rng.standard_normal((50, 128))
    assert np.allclose(label_scores(q, K, np.arange(128)), oracle.attention_scores(q, K), rtol=0, atol=1e-12)


def check_single_channel(label_scores):
    q = np.array([0.0, 2.0, -3.0, 0.5])
    K = np.array([[1.0, 1.5, 7.0, 9.0], [4.0, -2.0, 0.25, 3.0]])
    # channel 2 only: q_2 K[i, 2] = -3 * 7, -3 * 0.25
    assert np.allclose(label_scores(q, K, [2]), [-21.0, -0.75], rtol=0, atol=0)
    # channels {1, 3}: 2*1.5 + 0.5*9 = 7.5 ; 2*(-2) + 0.5*3 = -2.5
    assert np.allclose(label_scores(q, K, [1, 3]), [7.5, -2.5], rtol=0, atol=0)


def check_channel_order_irrelevant(label_scores):
    rng = np.random.default_rng(6)
    q, K = rng.standard_normal(128), rng.standard_normal((40, 128))
    c = np.array([3, 77, 12, 100, 5, 64, 90, 1])
    assert np.allclose(label_scores(q, K, c), label_scores(q, K, c[::-1].copy()), rtol=0, atol=1e-12)


def check_importance(channel_importance):
    # hand example: one query, two tokens, two channels
    Q = np.array([[2.0, -1.0]])
    K = np.array([[3.0, 4.0], [-1.0, 0.5]])
    # channel 0: |2*3| + |2*-1| = 8 ; channel 1: |-1*4| + |-1*0.5| = 4.5
    assert np.allclose(channel_importance(Q, K), [8.0, 4.5], rtol=0, atol=0)
    rng = np.random.default_rng(7)
    Q, K = rng.standard_normal((3, 6)), rng.standard_normal((5, 6))
    brute = np.zeros(6)
    for t in range(3):
        for i in range(5):
            for d in range(6):
                brute[d] += abs(Q[t, d] * K[i, d])
    assert np.allclose(channel_importance(Q, K), brute, rtol=1e-12, atol=0)


def check_choice(choose_channels):
    assert choose_channels([3.0, 1.0, 3.0, 2.0], 2).tolist() == [0, 2]
    assert choose_channels([1.0, 5.0, 5.0, 5.0], 2).tolist() == [1, 2]       # tie: lower indices
    assert choose_channels([9.0, 1.0, 2.0], 3).tolist() == [0, 1, 2]
    rng = np.random.default_rng(8)
    for _ in range(20):
        imp = rng.integers(0, 4, size=7).astype(float)    # many ties
        r = int(rng.integers(1, 8))
        best = None
        for sub in itertools.combinations(range(7), r):   # lexicographically smallest best subset
            key = sorted((-imp[d], d) for d in sub)
            if best is None or key < best[0]:
                best = (key, sub)
        assert choose_channels(imp, r).tolist() == sorted(best[1])


def test_label_pins_hold():
    check_all_channels_is_exact(oracle.label_scores)
    check_single_channel(oracle.label_scores)
    check_channel_order_irrelevant(oracle.label_scores)
    check_importance(oracle.channel_importance)
    check_choice(oracle.choose_channels)


def _fails(check, fn):
    try:
        check(fn)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name,check,mutant", [
    ("channel off by one", check_single_channel,
     lambda q, K, c: Lb.label_scores(q, K, np.asarray(c) + 1 if max(c) + 1 < len(q) else np.asarray(c))),
    ("all channels dropped one", check_all_channels_is_exact,
     lambda q, K, c: Lb.label_scores(q, K, np.asarray(c)[:-1])),
    ("importance without magnitudes", check_importance,
     lambda Q, K: np.asarray(Q).sum(axis=0) * np.asarray(K).sum(axis=0)),
    ("importance of keys only", check_importance,
     lambda Q, K: np.abs(np.asarray(K)).sum(axis=0)),
    ("ties to the higher channel", check_choice,
     lambda imp, r: np.sort(np.lexsort((-np.arange(len(imp)), -np.asarray(imp, float)))[:r])),
    ("smallest channels kept", check_choice,
     lambda imp, r: np.sort(np.lexsort((np.arange(len(imp)), np.asarray(imp, float)))[:r])),
])
def test_label_mutants_are_caught(name, check, mutant):
    assert _fails(check, mutant), name
