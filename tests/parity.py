"""Helpers that compare the CUDA path with the oracle on the same seeded inputs.

The oracle's inputs come from the host side of the workload generator only
(numpy Philox regeneration of the logical K/V rows); nothing the CUDA path
computes is fed to the oracle.  Index lists given to the GPU's sparse decode
are made by the generator (uniform / Zipf page runs) or by the oracle itself.
"""

from __future__ import annotations

import math
from functools import lru_cache
from typing import Dict, Iterable, List, Tuple

import numpy as np

import oracle
from top_sparse_decode_topk_b200 import workload as W

# Acceptance bars.  bf16 outputs: max-abs 5e-3 and rel-L2 2e-3; where bf16 rounding alone
# exceeds 5e-3 (|o| >= 2) the per-element bar is half a bf16 ulp plus 1e-4 |o|
# (oracle.elementwise_bar).  fp32 outputs: derived from the arithmetic (fp32
# accumulation and ex2.approx give relative errors ~1e-6 on outputs of size ~1).
BF16_MAX_ABS, BF16_REL_L2 = 5e-3, 2e-3
F32_MAX_ABS, F32_REL_L2 = 1e-4, 2e-5
LSE_ABS = 1e-3
TOPK_BAND = 1e-4


class OracleInputs:
    """Logical K/V rows of a workload regenerated on the host (cached per (b, g))."""

    def __init__(self, w: W.HostWorkload):
        self.w = w
        self._kv = {}

    def kv(self, b: int, g: int) -> Tuple[np.ndarray, np.ndarray]:
        key = (b, g)
        if key not in self._kv:
            K = oracle.from_bf16_bits(self.w.logical_kv_bits(b, g, "k"))
            V = oracle.from_bf16_bits(self.w.logical_kv_bits(b, g, "v"))
            self._kv[key] = (K, V)
        return self._kv[key]

    def q(self, t: int, h: int) -> np.ndarray:
        return oracle.from_bf16_bits(self.w.q_bits[t, h])

    def seq_of(self, t: int) -> int:
        return int(self.w.token_seq[t])

    def scores(self, t: int, h: int) -> np.ndarray:
        b = self.seq_of(t)
        g = h // self.w.cfg.group
        K, _ = self.kv(b, g)
        L = int(self.w.kv_len[t])
        return oracle.attention_scores(self.q(t, h), K[:L])

    def topk(self, t: int, h: int, k: int) -> np.ndarray:
        return oracle.exact_topk(self.scores(t, h), k)

    def attend(self, t: int, h: int, idx: np.ndarray, sm_scale: float):
        b = self.seq_of(t)
        g = h // self.w.cfg.group
        K, V = self.kv(b, g)
        L = int(self.w.kv_len[t])
        return oracle.sparse_attention(self.q(t, h), K[:L], V[:L], idx, sm_scale)

    def dense(self, t: int, h: int, sm_scale: float):
        b = self.seq_of(t)
        g = h // self.w.cfg.group
        K, V = self.kv(b, g)
        L = int(self.w.kv_len[t])
        return oracle.dense_attention(self.q(t, h), K[:L], V[:L], sm_scale)


def sample_pairs(w: W.HostWorkload, n_random: int, full_seqs: Iterable[int] = (0,), seed: int = 0) -> List[Tuple[int, int]]:
    """All (t, h) of the tokens of `full_seqs` plus n_random seeded other pairs."""
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    pairs = set()
    for b in full_seqs:
        for t in range(int(w.q_indptr[b]), int(w.q_indptr[b + 1])):
            for h in range(Hq):
                pairs.add((t, h))
    rng = np.random.default_rng(seed)
    for _ in range(n_random):
        pairs.add((int(rng.integers(T)), int(rng.integers(Hq))))
    return sorted(pairs)


def check_topk(inp: OracleInputs, gpu_idx: np.ndarray, gpu_count: np.ndarray, k_per_token: np.ndarray,
               pairs) -> Dict[str, int]:
    stats = {"lists": 0, "exact": 0, "band_only": 0}
    for t, h in pairs:
        k = int(k_per_token[t])
        s = inp.scores(t, h)
        ok, why = oracle.topk_sets_agree(gpu_idx[t, h], s, k, TOPK_BAND)
        assert ok, f"top-k (t={t}, h={h}, k={k}): {why}"
        n = min(k, s.shape[0])
        assert int(gpu_count[t, h]) == n
        stats["lists"] += 1
        ref = oracle.exact_topk(s, k)
        if np.array_equal(ref, gpu_idx[t, h][:n]):
            stats["exact"] += 1
        else:
            stats["band_only"] += 1
    return stats


def check_decode(inp: OracleInputs, idx: np.ndarray, out: np.ndarray, lse: np.ndarray, pairs, sm_scale: float,
                 out_is_bf16: bool, dense: bool = False) -> Tuple[float, float]:
    """Compare GPU rows with the oracle; returns the worst (max_abs, rel_l2)."""
    tol_abs, tol_rel = (BF16_MAX_ABS, BF16_REL_L2) if out_is_bf16 else (F32_MAX_ABS, F32_REL_L2)
    worst_abs = worst_rel = 0.0
    refs, gots = [], []
    for t, h in pairs:
        if dense:
            o_ref, lse_ref = inp.dense(t, h, sm_scale)
        else:
            o_ref, lse_ref = inp.attend(t, h, idx[t, h], sm_scale)
        o = out[t, h].astype(np.float64)
        ma, _ = oracle.output_errors(o, o_ref)
        worst_abs = max(worst_abs, ma)
        ok, why = oracle.output_within(o, o_ref, tol_abs, math.inf, out_is_bf16)
        assert ok, f"(t={t}, h={h}): {why}"
        refs.append(o_ref)
        gots.append(o)
        if lse is not None:
            if math.isinf(lse_ref):
                assert math.isinf(lse[t, h]) and lse[t, h] < 0, f"(t={t}, h={h}) lse {lse[t, h]} != -inf"
            else:
                assert abs(float(lse[t, h]) - lse_ref) <= LSE_ABS + 1e-5 * abs(lse_ref), \
                    f"(t={t}, h={h}) lse {lse[t, h]} vs {lse_ref}"
    if refs:
        _, rl = oracle.output_errors(np.stack(gots), np.stack(refs))
        worst_rel = rl
        assert rl <= tol_rel, f"rel-L2 {rl:.3g} > {tol_rel}"
    return worst_abs, worst_rel


def bf16_to_np(t) -> np.ndarray:
    """torch bf16/fp32 tensor (any device) -> float64 numpy (exact)."""
    import torch
    if t.dtype == torch.bfloat16:
        return oracle.from_bf16_bits(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.double().cpu().numpy()
