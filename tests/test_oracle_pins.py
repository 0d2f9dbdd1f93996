"""The oracle against facts outside itself, and proof that the pins bite.

Every check in oracle_pins.py runs on the real oracle and must pass.  Then a
set of deliberately broken copies of the oracle (each with one plausible
mistake: a flipped sign, a wrong tie rule, a dropped term, a missing max in the
log-sum-exp, a mis-applied scale, ...) is run through the same checks, and each
copy must fail at least one of them.  The mistakes live in this file only,
on the CPU.
"""

import numpy as np
import pytest

import oracle
from oracle import attention as A
from tests import oracle_pins as P


def test_golden_attention():
    P.check_golden_attention(oracle.sparse_attention)


def test_golden_topk():
    P.check_golden_topk(oracle.exact_topk)


def test_topk_brute_force():
    P.check_topk_brute_force(oracle.exact_topk)


def test_topk_invariants():
    P.check_topk_invariants(oracle.exact_topk)


def test_planted_needles_selected():
    P.check_planted_needles(oracle.exact_topk, oracle.attention_scores)


def test_dense_matches_library_sdpa():
    P.check_dense_matches_library(oracle.sparse_attention, oracle.dense_attention)


def test_k1_argmax_row():
    P.check_k1_argmax_row(oracle.sparse_attention, oracle.exact_topk, oracle.attention_scores)


def test_v_ones():
    P.check_v_ones(oracle.sparse_attention)


def test_permutation_invariance():
    P.check_permutation_invariance(oracle.sparse_attention)


def test_two_token_logistic():
    P.check_two_token_logistic(oracle.sparse_attention)


def test_split_merge_invariance():
    P.check_split_merge(oracle.sparse_attention)


def test_scores_exact_for_bf16_inputs():
    """For bf16 values of moderate magnitude (2^-8 <= |x| < 4, as in N(0,1) data)
    every product is exact and the 128-term float64 sum is exact: it equals an
    exact rational (Fraction) evaluation.  For arbitrary bf16 values the float64
    sum is within 128 float64 ulps of the largest partial sum of the exact one."""
    from fractions import Fraction
    rng = np.random.default_rng(11)

    def moderate(shape):
        mag = np.exp2(rng.uniform(-8, 2, size=shape)).astype(np.float32)
        x = mag * rng.choice([-1.0, 1.0], size=shape).astype(np.float32)
        u = x.view(np.uint32)
        return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)

    for trial in range(2):
        if trial == 0:
            bits_q, bits_k = moderate(128), moderate((4, 128))
        else:
            bits_q = rng.integers(0, 65536, size=128, dtype=np.uint16) & np.uint16(0xBFFF)
            bits_k = rng.integers(0, 65536, size=(4, 128), dtype=np.uint16) & np.uint16(0xBFFF)
        q = oracle.from_bf16_bits(bits_q)
        K = oracle.from_bf16_bits(bits_k)
        q[~np.isfinite(q)] = 0
        K[~np.isfinite(K)] = 0
        s = oracle.attention_scores(q, K)
        for r in range(4):
            terms = [Fraction(float(a)) * Fraction(float(b)) for a, b in zip(q, K[r])]
            exact = sum(terms)
            if trial == 0:
                assert Fraction(float(s[r])) == exact
            else:
                bound = 128 * 2.0 ** -52 * float(sum(abs(t) for t in terms))
                assert abs(float(Fraction(float(s[r])) - exact)) <= bound


# ---------------------------------------------------------------------------
# Mutants: each must fail at least one pin
# ---------------------------------------------------------------------------
def _topk_ascending(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    n = max(0, min(int(k), s.shape[0]))
    order = np.lexsort((np.arange(s.shape[0]), s))          # smallest instead of largest
    return np.sort(order[:n])


def _topk_ties_high(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    n = max(0, min(int(k), s.shape[0]))
    order = np.lexsort((-np.arange(s.shape[0]), -s))        # ties to the higher index
    return np.sort(order[:n])


def _topk_off_by_one(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    n = max(0, min(int(k), s.shape[0]))
    order = np.lexsort((np.arange(s.shape[0]), -s))
    return np.sort(order[:max(0, n - 1)])                   # drops one token


def _topk_unsorted(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    n = max(0, min(int(k), s.shape[0]))
    order = np.lexsort((np.arange(s.shape[0]), -s))
    return order[:n]                                         # score order, not token order


def _make_sparse(kind):
    def f(q, K, V, idx, sm_scale):
        q = np.asarray(q, dtype=np.float64)
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        idx = np.asarray(idx, dtype=np.int64).reshape(-1)
        if kind != "keep_padding":
            idx = idx[idx >= 0]
        if kind == "dedupe":
            idx = np.unique(idx)
        if kind == "drop_last" and idx.size > 1:
            idx = idx[:-1]
        D = V.shape[1]
        if idx.size == 0:
            return np.zeros(D), float("-inf")
        scale = 1.0 if kind == "no_scale" else sm_scale
        z = scale * (K[idx] @ q)
        if kind == "scale_squared":
            z = z * sm_scale
        m = np.max(z)
        w = np.exp(z - m)
        rows = K[idx] if kind == "weights_on_k" else V[idx]
        out = (w @ rows) / np.sum(w)
        lse = float(np.log(np.sum(w))) if kind == "lse_no_max" else float(m + np.log(np.sum(w)))
        if kind == "lse_log2":
            lse = float(m + np.log2(np.sum(w)))
        return out, lse
    return f


def _dense_from(sparse):
    return lambda q, K, V, s: sparse(q, K, V, np.arange(np.asarray(K).shape[0]), s)


TOPK_MUTANTS = {
    "ascending": _topk_ascending,
    "ties_high": _topk_ties_high,
    "off_by_one": _topk_off_by_one,
    "unsorted": _topk_unsorted,
}
SPARSE_MUTANTS = ["keep_padding", "dedupe", "drop_last", "no_scale", "scale_squared",
                  "weights_on_k", "lse_no_max", "lse_log2"]


def test_real_oracle_passes_all_pins():
    assert P.run_all(oracle.sparse_attention, oracle.dense_attention,
                     oracle.exact_topk, oracle.attention_scores) == []


@pytest.mark.parametrize("name", sorted(TOPK_MUTANTS))
def test_topk_mutant_is_caught(name):
    failed = P.run_all(oracle.sparse_attention, oracle.dense_attention,
                       TOPK_MUTANTS[name], oracle.attention_scores)
    assert failed, f"topk mutant {name} passed every pin"


@pytest.mark.parametrize("kind", SPARSE_MUTANTS)
def test_attention_mutant_is_caught(kind):
    sp = _make_sparse(kind)
    failed = P.run_all(sp, _dense_from(sp), oracle.exact_topk, oracle.attention_scores)
    assert failed, f"attention mutant {kind} passed every pin"


def test_scores_transposed_operand_is_caught():
    # q against the wrong axis of K: with L != D this raises or mis-shapes.
    def bad_scores(q, K):
        K = np.asarray(K, dtype=np.float64)
        return (K.T @ np.resize(q, K.shape[0]))[: K.shape[0]]
    failed = P.run_all(oracle.sparse_attention, oracle.dense_attention, oracle.exact_topk, bad_scores)
    assert failed
