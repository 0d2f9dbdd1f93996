"""The acceptance rules themselves (CPU): oracle/compare.py against hand-made cases.

Every GPU parity test passes or fails through `topk_sets_agree` (a top-k list against
the exact selection, with the float32 band) and `output_within` / `output_errors`
(a decode output against the float64 result).  The cases below are worked out by
hand from the rules' definitions, so that the rules are pinned to something other
than themselves.  Then each rule is re-created with one plausible mistake planted in
its source text (the k-th score taken as the largest, an absolute band, a one-sided
set difference, a missing count or padding check, the relative L2 error divided by
the wrong norm, the bf16 allowance added on top of 5e-3 ...), and every such copy
must fail at least one case.  The mistakes live in this file only, on the CPU.
"""

import inspect
import math
import textwrap

import numpy as np
import pytest

import oracle
from oracle import compare as C

# --------------------------------------------------------------------------------------
# top-k acceptance
# --------------------------------------------------------------------------------------
# L = 10 scores.  Exact top-4 (ties to the lower index): 9.0 (token 1), 8.0 (6), 7.0 (3),
# 3.0 (9), so s_k = 3.0 and the band is 1e-4 * 3 = 3e-4.  Token 4 (2.9998) lies inside the
# band, token 7 (2.9990) outside it.
S10 = [0.5, 9.0, 2.0, 7.0, 2.9998, 1.0, 8.0, 2.9990, 0.0, 3.0]
TOPK_CASES = [
    # (name, scores, k, gpu list, accepted?)
    ("exact set", S10, 4, [1, 3, 6, 9], True),
    ("exact set with padding", S10, 4, [1, 3, 6, 9, -1, -1], True),
    ("swap with a token inside the band", S10, 4, [1, 3, 4, 6], True),
    ("swap with a token just outside the band", S10, 4, [1, 3, 6, 7], False),
    # the dropped token (8.0) is far outside the band, the added one (2.9998) inside it
    ("a high-score token dropped for an in-band one", S10, 4, [1, 3, 4, 9], False),
    ("count too small", S10, 4, [1, 3, 6, -1], False),
    ("count too large", S10, 4, [1, 3, 4, 6, 9], False),
    ("duplicate entry", S10, 4, [1, 3, 3, 6], False),
    ("descending order", S10, 4, [9, 6, 3, 1], False),
    ("junk after the -1 padding", S10, 4, [1, 3, 6, 9, -1, 5], False),
    ("a negative non-padding value after the list", S10, 4, [1, 3, 6, 9, -1, -7], False),
    # a buffer shorter than k: the missing token (9, at s_k itself) is inside the band, so
    # only the count rejects it
    ("list shorter than k", S10, 4, [1, 3, 6], False),
    ("-1 inside the valid prefix", S10, 4, [1, -1, 3, 6, 9, -1], False),
    ("index past the context", S10, 4, [1, 3, 6, 10], False),
    # k > L: every token, padded
    ("k > L keeps all tokens", [2.0, 1.0, 3.0], 5, [0, 1, 2, -1, -1], True),
    ("k > L with a token missing", [2.0, 1.0, 3.0], 5, [0, 2, -1, -1, -1], False),
    ("k = 0", [2.0, 1.0, 3.0], 0, [-1, -1], True),
    ("k = 0 with an entry", [2.0, 1.0, 3.0], 0, [1, -1], False),
    # negative k-th score: s = [-1, -3, -2, -2.0001, -5], k = 2 -> {0, 2}, s_k = -2, band 2e-4
    ("negative s_k, in-band swap", [-1.0, -3.0, -2.0, -2.0001, -5.0], 2, [0, 3], True),
    ("negative s_k, out-of-band swap", [-1.0, -3.0, -2.0, -2.0001, -5.0], 2, [0, 1], False),
    # exact ties at s_k are inside the band (the tie order is pinned index for index by the
    # GPU tie tests, not by this rule)
    ("tie at s_k resolved to the higher index", [1.0, 2.0, 2.0, 2.0, 0.0], 2, [1, 3], True),
    # the band is centred on the k-th score, not the (k+1)-th: s_k = 3.0 (band [2.9997, 3.0003]),
    # s_(k+1) = 2.99985; token 3 (2.9996) is within 3e-4 of s_(k+1) but not of s_k
    ("swap outside the band of s_k, inside one around s_(k+1)", [5.0, 3.0, 2.99985, 2.9996, 0.0], 2, [0, 3],
     False),
    # the band is relative: a large s_k widens it.  s_k = 1000, band 0.1: 999.95 is inside.
    ("relative band at a large s_k", [1000.0, 999.95, 5.0, 2000.0], 2, [1, 3], True),
    ("relative band at a large s_k, outside", [1000.0, 999.8, 5.0, 2000.0], 2, [1, 3], False),
]


def _run_topk_cases(fn):
    for name, s, k, g, want in TOPK_CASES:
        ok, why = fn(np.array(g, dtype=np.int32), np.array(s, dtype=np.float64), k, 1e-4)
        assert bool(ok) == want, f"{name}: got {ok} ({why})"


def test_topk_rule_on_hand_made_cases():
    _run_topk_cases(oracle.topk_sets_agree)


# --------------------------------------------------------------------------------------
# decode output acceptance
# --------------------------------------------------------------------------------------
def test_output_errors_hand_example():
    # d = [0, 0, -1]: max-abs 1; rel-L2 = |d| / |ref| = 1 / sqrt(1 + 4 + 16)
    ma, rl = oracle.output_errors([1.0, 2.0, 3.0], [1.0, 2.0, 4.0])
    assert ma == 1.0
    assert abs(rl - 1.0 / math.sqrt(21.0)) < 1e-15
    # the sign of the difference does not matter
    ma2, rl2 = oracle.output_errors([1.0, 2.0, 5.0], [1.0, 2.0, 4.0])
    assert ma2 == 1.0 and abs(rl2 - 1.0 / math.sqrt(21.0)) < 1e-15
    # a zero reference: the absolute L2 norm of the difference
    ma3, rl3 = oracle.output_errors([3.0, 4.0], [0.0, 0.0])
    assert ma3 == 4.0 and rl3 == 5.0
    assert oracle.output_errors([], []) == (0.0, 0.0)


def test_bf16_half_ulp():
    assert oracle.bf16_half_ulp(np.array([1.0]))[0] == 2 ** -8
    assert oracle.bf16_half_ulp(np.array([1.99]))[0] == 2 ** -8
    assert oracle.bf16_half_ulp(np.array([-2.5]))[0] == 2 ** -7
    assert oracle.bf16_half_ulp(np.array([0.3]))[0] == 2 ** -10
    # every bf16 value in [1, 4) is a whole number of ulps (2 half ulps)
    xs = np.concatenate([np.arange(128, 256) * 2.0 ** -7, np.arange(128, 256) * 2.0 ** -6])
    assert np.all(np.mod(xs, 2 * oracle.bf16_half_ulp(xs)) == 0)


OUT_CASES = [
    # (name, out, ref, bf16?, accepted?)
    ("within 5e-3", [0.5049], [0.5], True, True),
    ("just over 5e-3 below |o| = 2", [0.5051], [0.5], True, False),
    ("within 5e-3 at |o| = 1.9", [1.9049], [1.9], True, True),
    ("just over 5e-3 at |o| = 1.9", [1.9051], [1.9], True, False),
    # |o| = 3: half ulp 2^-7 = 0.0078125, plus 1e-4 * 3 = 0.0003: bar 0.0081125
    ("half an ulp plus the fp32 budget at |o| = 3", [3.0081], [3.0], True, True),
    ("beyond half an ulp plus the budget at |o| = 3", [3.0082], [3.0], True, False),
    # the old additive bar (5e-3 + half ulp = 0.0128 at |o| = 3) would accept this
    ("5e-3 on top of half an ulp is not granted", [3.012], [3.0], True, False),
    ("fp32 outputs: the absolute bar only", [3.0002], [3.0], False, False),
    ("fp32 outputs within 1e-4", [3.00009], [3.0], False, True),
    ("negative values are symmetric", [-3.0081], [-3.0], True, True),
    ("a NaN never passes", [float("nan")], [0.0], True, False),
]


def _run_output_cases(within):
    for name, o, r, bf, want in OUT_CASES:
        tol = 5e-3 if bf else 1e-4
        ok, why = within(np.array(o), np.array(r), tol, math.inf, bf)
        assert bool(ok) == want, f"{name}: got {ok} ({why})"
    # the rel-L2 bar on a unit-norm block: errors of 1e-3 on n elements give sqrt(n) 1e-3,
    # which passes 2e-3 for n = 3 and fails it for n = 5 (each element within max-abs)
    ref = np.zeros(16)
    ref[0] = 1.0
    out = ref.copy()
    out[1:4] += 1e-3
    ok, why = within(out, ref, 5e-3, 2e-3, True)
    assert ok, why
    out[4:6] += 1e-3
    ok, _ = within(out, ref, 5e-3, 2e-3, True)
    assert not ok
    # a uniform relative error: 1.5e-3 passes, 3e-3 does not
    ref2 = np.full(4, 1.0)
    ok, why = within(ref2 * (1 + 1.5e-3), ref2, 5e-3, 2e-3, True)
    assert ok, why
    ok, _ = within(ref2 * (1 + 3e-3), ref2, 5e-3, 2e-3, True)
    assert not ok


def test_output_rule_on_hand_made_cases():
    _run_output_cases(oracle.output_within)


# --------------------------------------------------------------------------------------
# planted mistakes: each must be caught
# --------------------------------------------------------------------------------------
def _mutant(fn, old: str, new: str):
    """`fn` re-created from its source with `old` replaced by `new` (exactly once)."""
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, f"mutation site {old!r} not found once in {fn.__name__}"
    env = dict(vars(C))
    exec(compile(src.replace(old, new), f"<mutant of {fn.__name__}>", "exec"), env)
    return env[fn.__name__]


TOPK_MUTANTS = [
    ("s_k taken as the largest score", "sk = np.sort(s)[::-1][n - 1]", "sk = np.sort(s)[::-1][0]"),
    ("s_k taken as the (k+1)-th score", "sk = np.sort(s)[::-1][n - 1]", "sk = np.sort(s)[::-1][min(n, L - 1)]"),
    ("absolute band", "band = rel_band * abs(sk)", "band = rel_band"),
    ("signed band", "band = rel_band * abs(sk)", "band = rel_band * sk"),
    ("one-sided difference (missing exact tokens only)", "diff = np.setxor1d(ref, valid)",
     "diff = np.setdiff1d(ref, valid)"),
    ("one-sided difference (extra GPU tokens only)", "diff = np.setxor1d(ref, valid)",
     "diff = np.setdiff1d(valid, ref)"),
    ("no count check", "if valid.size != n:", "if False:"),
    ("no padding check", "if np.any(g[n:] != -1):", "if False:"),
    ("duplicates allowed", "np.diff(valid) <= 0", "np.diff(valid) < 0"),
    ("no order check", "if np.any(np.diff(valid) <= 0):", "if False:"),
    ("band around the score of the highest kept index", "sk = np.sort(s)[::-1][n - 1]", "sk = s[ref[-1]]"),
]


@pytest.mark.parametrize("name,old,new", TOPK_MUTANTS, ids=[m[0] for m in TOPK_MUTANTS])
def test_topk_rule_mutants_are_caught(name, old, new):
    bad = _mutant(C.topk_sets_agree, old, new)
    with pytest.raises((AssertionError, IndexError, ValueError)):
        _run_topk_cases(bad)


OUTPUT_MUTANTS = [
    # (name, function, old, new)
    ("rel-L2 over the output's norm", C.output_errors, "nr = float(np.linalg.norm(r))",
     "nr = float(np.linalg.norm(o))"),
    ("rel-L2 over the squared norm", C.output_errors, "rel = float(np.linalg.norm(d) / nr)",
     "rel = float(np.linalg.norm(d) / nr ** 2)"),
    ("signed max instead of max-abs", C.output_errors, "max_abs = float(np.max(np.abs(d)))",
     "max_abs = float(np.max(d))"),
    ("mean-abs instead of max-abs", C.output_errors, "max_abs = float(np.max(np.abs(d)))",
     "max_abs = float(np.mean(np.abs(d)))"),
]


@pytest.mark.parametrize("name,fn,old,new", OUTPUT_MUTANTS, ids=[m[0] for m in OUTPUT_MUTANTS])
def test_output_errors_mutants_are_caught(name, fn, old, new):
    bad = _mutant(fn, old, new)
    with pytest.raises(AssertionError):
        _output_errors_cases(bad)


def _output_errors_cases(output_errors):
    ma, rl = output_errors([1.0, 2.0, 3.0], [1.0, 2.0, 4.0])
    assert ma == 1.0 and abs(rl - 1.0 / math.sqrt(21.0)) < 1e-15
    ma2, rl2 = output_errors([1.0, 2.0, 5.0], [1.0, 2.0, 4.0])
    assert ma2 == 1.0 and abs(rl2 - 1.0 / math.sqrt(21.0)) < 1e-15
    ma3, rl3 = output_errors([3.0, 4.0], [0.0, 0.0])
    assert ma3 == 4.0 and rl3 == 5.0


def test_output_errors_cases_pass_on_the_rule():
    _output_errors_cases(oracle.output_errors)


BAR_MUTANTS = [
    ("5e-3 added on top of the half ulp", C.elementwise_bar,
     "np.maximum(float(max_abs), bf16_half_ulp(r) + FP32_EVAL_REL * np.abs(r))",
     "float(max_abs) + bf16_half_ulp(r)"),
    ("a whole ulp", C.elementwise_bar,
     "np.maximum(float(max_abs), bf16_half_ulp(r) + FP32_EVAL_REL * np.abs(r))",
     "np.maximum(float(max_abs), 2 * bf16_half_ulp(r))"),
    ("the bf16 allowance applied to fp32 outputs", C.elementwise_bar, "if not bf16_rounded:", "if False:"),
    ("no bf16 allowance", C.elementwise_bar,
     "np.maximum(float(max_abs), bf16_half_ulp(r) + FP32_EVAL_REL * np.abs(r))",
     "np.full(r.shape, float(max_abs))"),
    ("half ulp one binade low", C.bf16_half_ulp, "np.exp2(e - 8)", "np.exp2(e - 9)"),
]


@pytest.mark.parametrize("name,fn,old,new", BAR_MUTANTS, ids=[m[0] for m in BAR_MUTANTS])
def test_bar_mutants_are_caught(name, fn, old, new):
    env = dict(vars(C))
    env[fn.__name__] = _mutant(fn, old, new)
    if fn is C.bf16_half_ulp:   # elementwise_bar must see the planted helper too
        env["elementwise_bar"] = _rebind(C.elementwise_bar, env)
    within = _rebind(C.output_within, env)   # output_within calling the planted helper
    with pytest.raises(AssertionError):
        _run_output_cases(within)


def test_within_mutants_are_caught():
    for old, new in (("if rel > rel_l2:", "if False:"),
                     ("if excess.size and np.max(excess) > 0:", "if False:"),
                     ("if not np.all(np.isfinite(o)):", "if False:")):
        bad = _mutant(C.output_within, old, new)
        with pytest.raises(AssertionError):
            _run_output_cases(bad)


def _rebind(fn, env):
    src = textwrap.dedent(inspect.getsource(fn))
    g = dict(env)
    exec(compile(src, f"<rebound {fn.__name__}>", "exec"), g)
    return g[fn.__name__]
