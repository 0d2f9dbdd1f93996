"""Seeded synthetic decode workloads for context-sparse decode attention.

This module only produces inputs. It holds none of the attention arithmetic
(no dot products, softmax or selection): both the CUDA path and the CPU oracle
receive what it makes, and neither is imported here.

What the workloads imitate ("Inference Time Context Sparsity: Illusion or
Opportunity?", gist.science technical summary, sections 2 and 3.C): decode
steps over 32K-128K contexts with about 2% of the tokens kept (50x sparsity),
with the kept set free to differ per token, per query and per head.  The
evaluation suites the pages name (RULER-HARD, LOFT, AIME 2025, SWE-Bench) are
not used; seeded random tensors of the same shapes stand in for them.

Random values
-------------
* Bulk K/V/q elements come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
  "Parallel random numbers: as easy as 1, 2, 3", SC 2011), a counter-based
  generator: element (tensor, b, g, i, d) -> one 16-bit lane of one Philox
  output word.  The 16-bit uniform u maps to a bf16 value through a fixed
  table of standard-normal quantiles, table[u] = bf16(Phi^-1((u + 0.5) / 2^16)).
  The host (numpy) and the device fill kernel (``csrc/workload_fill.cu``)
  implement the same definition, so any element can be regenerated on the
  host without touching the rest of a multi-GB cache.
* Small structured pieces (page permutation, sequence lengths, needle
  positions, planted key rows, index lists) come from numpy's PCG64 seeded by
  a SeedSequence of (seed, config, purpose); they are made on the host once and
  shared by both sides.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# --------------------------------------------------------------------------
# Philox4x32-10 (published definition: SC 2011 paper above, Random123 docs)
# --------------------------------------------------------------------------
PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)

TENSOR_K = 1
TENSOR_V = 2
TENSOR_Q = 3

HEAD_DIM = 128
# Poison written into cache slots that belong to no token (tail of a last page,
# unmapped pages).  Any kernel that reads such a slot by mistake visibly skews
# its output: keys score large, values are far outside N(0,1).
POISON_K = 4.0
POISON_V = 1000.0


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds on uint32 arrays; returns four uint32 arrays."""
    c0 = np.asarray(c0, dtype=np.uint64) & _MASK32
    c1 = np.asarray(c1, dtype=np.uint64) & _MASK32
    c2 = np.asarray(c2, dtype=np.uint64) & _MASK32
    c3 = np.asarray(c3, dtype=np.uint64) & _MASK32
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    c0 = c0.copy(); c1 = c1.copy(); c2 = c2.copy(); c3 = c3.copy()
    key0 = k0 & 0xFFFFFFFF
    key1 = k1 & 0xFFFFFFFF
    for _ in range(10):
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        hi0 = p0 >> np.uint64(32)
        lo0 = p0 & _MASK32
        hi1 = p1 >> np.uint64(32)
        lo1 = p1 & _MASK32
        n0 = hi1 ^ c1 ^ np.uint64(key0)
        n2 = hi0 ^ c3 ^ np.uint64(key1)
        c0, c1, c2, c3 = n0, lo1, n2, lo0
        key0 = (key0 + PHILOX_W0) & 0xFFFFFFFF
        key1 = (key1 + PHILOX_W1) & 0xFFFFFFFF
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))


# --------------------------------------------------------------------------
# bf16 bit helpers (storage format only)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


_NORMAL_TABLE: Optional[np.ndarray] = None


def normal_table() -> np.ndarray:
    """uint16[65536] bf16 bits of the standard-normal quantile at (u + 0.5) / 2^16."""
    global _NORMAL_TABLE
    if _NORMAL_TABLE is None:
        from scipy.special import ndtri
        p = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
        _NORMAL_TABLE = f32_to_bf16_bits(ndtri(p).astype(np.float32))
    return _NORMAL_TABLE


def _lanes16(words: Sequence[np.ndarray]) -> np.ndarray:
    """Split four uint32 Philox words into eight uint16 lanes (low half first)."""
    out = np.empty(words[0].shape + (8,), dtype=np.uint16)
    for j, w in enumerate(words):
        out[..., 2 * j] = (w & 0xFFFF).astype(np.uint16)
        out[..., 2 * j + 1] = (w >> 16).astype(np.uint16)
    return out


def kv_base_bits(seed: int, tensor_id: int, b: int, g: int, tokens: np.ndarray) -> np.ndarray:
    """bf16 bits [len(tokens), 128] of the unplanted K or V rows of (sequence b, kv head g).

    Counter of element d of token i: (i, d//8 + 16*g + 65536*b, tensor_id, 0),
    key (seed low word, seed high word); lane d%8 of the output picks the value.
    """
    tokens = np.asarray(tokens, dtype=np.uint64)
    blk = np.arange(16, dtype=np.uint64)
    c0 = tokens[:, None]
    c1 = blk[None, :] + np.uint64(16 * g + 65536 * b)
    words = philox4x32_10(c0, c1, np.uint64(tensor_id), np.uint64(0), seed & 0xFFFFFFFF, seed >> 32)
    u = _lanes16(words)                      # [n, 16, 8]
    return normal_table()[u].reshape(len(tokens), HEAD_DIM)


def q_base_bits(seed: int, num_tokens: int, num_heads: int) -> np.ndarray:
    """bf16 bits [T, Hq, 128] of the queries: counter (t, d//8 + 16*h, TENSOR_Q, 0)."""
    t = np.arange(num_tokens, dtype=np.uint64)[:, None, None]
    h = np.arange(num_heads, dtype=np.uint64)[None, :, None]
    blk = np.arange(16, dtype=np.uint64)[None, None, :]
    words = philox4x32_10(t, blk + np.uint64(16) * h, np.uint64(TENSOR_Q), np.uint64(0),
                          seed & 0xFFFFFFFF, seed >> 32)
    u = _lanes16(words)                      # [T, Hq, 16, 8]
    return normal_table()[u].reshape(num_tokens, num_heads, HEAD_DIM)


# --------------------------------------------------------------------------
# Configurations (shapes of the pages' 32K-128K, ~50x-sparsity decode study)
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: Optional[int] = None                 # fixed context length N
    seq_len_range: Optional[Tuple[int, int]] = None  # inclusive uniform range (ragged)
    tokens_per_seq: int = 1                       # decode queries per sequence
    layout: str = "paged"                         # "paged" (HND pages) or "contiguous"
    page_size: int = 16
    ks: Tuple[int, ...] = ()                      # fixed k values (first one is the default)
    k_frac_ceil: Optional[float] = None           # k = ceil(frac * kv_len) per token
    planted: bool = False                         # needles + sink + recent window
    causal: bool = True
    out_dtype: str = "bf16"
    index_mode: str = "topk"                      # "topk", "uniform" or "zipf"
    description: str = ""

    @property
    def head_dim(self) -> int:
        return HEAD_DIM

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def num_tokens(self) -> int:
        return self.batch * self.tokens_per_seq

    @property
    def max_seq_len(self) -> int:
        return self.seq_len if self.seq_len is not None else self.seq_len_range[1]


def k_for_sparsity(n: int, x: float) -> int:
    """k kept at x-fold sparsity: round-half-up of n/x, at least 1 (4096/50 -> 82)."""
    return max(1, int(math.floor(n / x + 0.5)))


CONFIGS: Dict[str, DecodeConfig] = {
    "tiny": DecodeConfig(
        name="tiny", batch=1, num_q_heads=8, num_kv_heads=2, seq_len=4096,
        layout="contiguous", ks=(82,), out_dtype="f32", planted=False,
        description="batch 1, 8/2 heads, N=4096, k=82, contiguous, iid N(0,1), fp32 out"),
    "llama3_8b": DecodeConfig(
        name="llama3_8b", batch=8, num_q_heads=32, num_kv_heads=8, seq_len=32768,
        ks=(655,), planted=True,
        description="batch 8, 32/8 heads, N=32768, k=655, paged (16), needles/sink/window"),
    "qwen25_72b": DecodeConfig(
        name="qwen25_72b", batch=4, num_q_heads=64, num_kv_heads=8, seq_len=131072,
        ks=(2621, 13107, 1311), planted=True,
        description="batch 4, 64/8 heads, N=131072, k=N/50 (also N/10, N/100), paged (16)"),
    "ragged": DecodeConfig(
        name="ragged", batch=32, num_q_heads=32, num_kv_heads=8, seq_len_range=(8192, 131072),
        tokens_per_seq=4, k_frac_ceil=0.02, planted=True,
        description="32 seqs, len U[8192,131072], 4 causal decode queries each, 32/8 heads, "
                    "k=ceil(0.02*kv_len), paged (16)"),
    "sweep": DecodeConfig(
        name="sweep", batch=16, num_q_heads=32, num_kv_heads=8, seq_len=65536,
        ks=tuple(k_for_sparsity(65536, x) for x in (1, 4, 10, 25, 50, 100, 200)),
        index_mode="uniform", planted=False,
        description="batch 16, 32/8 heads, N=65536, k in {N..N/200}, uniform or Zipf page-run indices"),
    # reduced copies of two shapes above, small enough for detailed profiler captures (a few GB
    # on the device) while the rows the sparse kernel reads still exceed the 126 MB L2
    "qwen25_72b_b2": DecodeConfig(
        name="qwen25_72b_b2", batch=2, num_q_heads=64, num_kv_heads=8, seq_len=131072,
        ks=(2621,), planted=True,
        description="the Qwen2.5-72B shape with batch 2: 64/8 heads, N=131072, k=2621, paged (16)"),
    "ragged_8": DecodeConfig(
        name="ragged_8", batch=8, num_q_heads=32, num_kv_heads=8, seq_len_range=(8192, 131072),
        tokens_per_seq=4, k_frac_ceil=0.02, planted=True,
        description="the ragged batch with 8 seqs: len U[8192,131072], 4 causal decode queries each, "
                    "32/8 heads, k=ceil(0.02*kv_len), paged (16)"),
}

CONFIG_IDS = {"tiny": 1, "llama3_8b": 2, "qwen25_72b": 3, "ragged": 4, "sweep": 5, "qwen25_72b_b2": 6,
              "ragged_8": 7}


# --------------------------------------------------------------------------
# Host-side workload description
# --------------------------------------------------------------------------
@dataclass
class HostWorkload:
    cfg: DecodeConfig
    seed: int
    seq_lens: np.ndarray            # int32 [B]
    q_indptr: np.ndarray            # int32 [B+1]
    token_seq: np.ndarray           # int32 [T]  sequence of each query token
    kv_len: np.ndarray              # int32 [T]  tokens visible to each query
    q_bits: np.ndarray              # uint16 [T, Hq, 128]
    page_table: np.ndarray          # int32 [B, max_pages_per_seq]
    num_pages: int                  # physical pages per tensor (paged) or B (contiguous)
    page_size: int                  # 16, or max_seq_len for the contiguous layout
    # planted key rows: (b, g) -> (token positions int64[n], bf16 bits uint16[n, 128])
    planted_k: Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]] = field(default_factory=dict)

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.page_table.shape[1])

    def k_per_token(self, k: Optional[int] = None) -> np.ndarray:
        """int32 [T]: the k of each query token (fixed k, or the ceil-fraction rule)."""
        if self.cfg.k_frac_ceil is not None and k is None:
            return np.array([int(math.ceil(self.cfg.k_frac_ceil * L - 1e-12)) for L in self.kv_len],
                            dtype=np.int32)
        kk = self.cfg.ks[0] if k is None else k
        return np.full(len(self.kv_len), kk, dtype=np.int32)

    def logical_kv_bits(self, b: int, g: int, which: str, tokens: Optional[np.ndarray] = None) -> np.ndarray:
        """bf16 bits of the K ('k') or V ('v') rows of (sequence b, kv head g) at `tokens`."""
        L = int(self.seq_lens[b])
        if tokens is None:
            tokens = np.arange(L, dtype=np.int64)
        tokens = np.asarray(tokens, dtype=np.int64)
        tid = TENSOR_K if which == "k" else TENSOR_V
        rows = kv_base_bits(self.seed, tid, b, g, tokens)
        if which == "k" and (b, g) in self.planted_k:
            pos, bits = self.planted_k[(b, g)]
            where = {int(p): j for j, p in enumerate(pos)}
            for r, t in enumerate(tokens):
                j = where.get(int(t))
                if j is not None:
                    rows[r] = bits[j]
        return rows

    def physical_row(self, b: int, g: int, i: int) -> int:
        """Row number (units of 128 elements) of token i of (b, g) in the cache tensor."""
        page = int(self.page_table[b, i // self.page_size])
        return (page * self.cfg.num_kv_heads + g) * self.page_size + (i % self.page_size)


def _rng(seed: int, cfg: DecodeConfig, purpose: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, CONFIG_IDS.get(cfg.name, 0), purpose]))


def _unit(v: np.ndarray) -> np.ndarray:
    return v / np.linalg.norm(v)


def _random_unit_orthogonal(rng: np.random.Generator, ref: np.ndarray) -> np.ndarray:
    z = rng.standard_normal(ref.shape[0])
    z = z - (z @ ref) * ref
    return _unit(z)


def make_workload(cfg: DecodeConfig, seed: int = 0, seq_lens: Optional[Sequence[int]] = None) -> HostWorkload:
    """Build the host-side description of one seeded workload (no bulk K/V).

    `seq_lens` overrides the configuration's lengths (each <= cfg.max_seq_len).
    """
    B, Hq, Hkv, G = cfg.batch, cfg.num_q_heads, cfg.num_kv_heads, cfg.group
    if seq_lens is not None:
        seq_lens = np.asarray(seq_lens, dtype=np.int32)
        assert seq_lens.shape == (B,) and int(seq_lens.max()) <= cfg.max_seq_len
    elif cfg.seq_len is not None:
        seq_lens = np.full(B, cfg.seq_len, dtype=np.int32)
    else:
        lo, hi = cfg.seq_len_range
        seq_lens = _rng(seed, cfg, 1).integers(lo, hi + 1, size=B).astype(np.int32)
    Tb = cfg.tokens_per_seq
    q_indptr = (np.arange(B + 1, dtype=np.int32) * Tb).astype(np.int32)
    token_seq = np.repeat(np.arange(B, dtype=np.int32), Tb)
    # query j of the n_b tokens of sequence b sees kv_len = L_b - n_b + j + 1 (causal)
    kv_len = np.empty(B * Tb, dtype=np.int32)
    for b in range(B):
        for j in range(Tb):
            kv_len[b * Tb + j] = seq_lens[b] - Tb + j + 1 if cfg.causal else seq_lens[b]
    q_bits = q_base_bits(seed, B * Tb, Hq)

    if cfg.layout == "contiguous":
        page_size = cfg.max_seq_len
        page_table = np.arange(B, dtype=np.int32)[:, None]
        num_pages = B
    else:
        page_size = cfg.page_size
        max_pages = -(-cfg.max_seq_len // page_size)
        pages_per_seq = [-(-int(L) // page_size) for L in seq_lens]
        num_pages = int(sum(pages_per_seq))
        perm = _rng(seed, cfg, 2).permutation(num_pages).astype(np.int32)
        page_table = np.full((B, max_pages), -1, dtype=np.int32)
        off = 0
        for b, n in enumerate(pages_per_seq):
            page_table[b, :n] = perm[off:off + n]
            off += n

    w = HostWorkload(cfg=cfg, seed=seed, seq_lens=seq_lens, q_indptr=q_indptr,
                     token_seq=token_seq, kv_len=kv_len, q_bits=q_bits,
                     page_table=page_table, num_pages=num_pages, page_size=page_size)
    if cfg.planted:
        _plant(w, _rng(seed, cfg, 3))
    return w


def _plant(w: HostWorkload, rng: np.random.Generator) -> None:
    """Needles, boosted sink and recent window in the keys (reading of the configs).

    * 64 needle positions per sequence, uniform without replacement in
      [1, L-128).  Needle j of kv head g gets K = sqrt(D) (0.5 qhat + sqrt(0.75) u)
      where qhat is the unit query of the (j mod G)-th q head of the group and
      u a random unit vector orthogonal to it (cosine 0.5 with that query).
    * token 0 (sink): K = 2 sqrt(D) (0.9 mhat + sqrt(0.19) u), mhat the unit mean of
      the group's queries.
    * last 128 tokens (recent window): K = sqrt(D) (0.5 mhat + sqrt(0.75) u_i).
    The queries used are those of the first decode token of the sequence.
    """
    cfg = w.cfg
    D, G = HEAD_DIM, cfg.group
    sd = math.sqrt(D)
    q = bf16_bits_to_f64(w.q_bits)
    for b in range(cfg.batch):
        L = int(w.seq_lens[b])
        t0 = int(w.q_indptr[b])
        needles = np.sort(rng.choice(np.arange(1, L - 128), size=64, replace=False))
        for g in range(cfg.num_kv_heads):
            heads = [g * G + j for j in range(G)]
            qhat = [_unit(q[t0, h]) for h in heads]
            mhat = _unit(np.mean([q[t0, h] for h in heads], axis=0))
            pos, rows = [], []
            for j, p in enumerate(needles):
                qh = qhat[j % G]
                rows.append(sd * (0.5 * qh + math.sqrt(0.75) * _random_unit_orthogonal(rng, qh)))
                pos.append(int(p))
            rows.append(2.0 * sd * (0.9 * mhat + math.sqrt(0.19) * _random_unit_orthogonal(rng, mhat)))
            pos.append(0)
            for i in range(L - 128, L):
                rows.append(sd * (0.5 * mhat + math.sqrt(0.75) * _random_unit_orthogonal(rng, mhat)))
                pos.append(i)
            w.planted_k[(b, g)] = (np.array(pos, dtype=np.int64),
                                   f32_to_bf16_bits(np.array(rows, dtype=np.float32)))


# --------------------------------------------------------------------------
# Supplied index lists (sparsity sweep): uniform scatter and Zipf page runs
# --------------------------------------------------------------------------
def uniform_indices(w: HostWorkload, k: int, seed_purpose: int = 10) -> np.ndarray:
    """int32 [T, Hq, k]: per (t, h) k distinct tokens of [0, kv_len) uniformly, ascending.

    Lists shorter than k (kv_len < k) are padded with -1.
    """
    rng = _rng(w.seed, w.cfg, seed_purpose + k)
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    out = np.full((T, Hq, k), -1, dtype=np.int32)
    for t in range(T):
        L = int(w.kv_len[t])
        n = min(k, L)
        for h in range(Hq):
            if n == L:
                out[t, h, :n] = np.arange(L, dtype=np.int32)
            else:
                out[t, h, :n] = np.sort(rng.choice(L, size=n, replace=False)).astype(np.int32)
    return out


def zipf_page_run_indices(w: HostWorkload, k: int, alpha: float = 1.1, seed_purpose: int = 20) -> np.ndarray:
    """int32 [T, Hq, k]: clustered lists made of whole 16-token page runs.

    Per sequence the logical pages are permuted once (seeded); per (t, h) page
    ranks r = 1..P are drawn without replacement with probability proportional
    to r^-alpha and whole pages are taken in draw order until k tokens are
    reached (the last page drawn gives its lowest slots only).  Ascending.
    """
    rng = _rng(w.seed, w.cfg, seed_purpose + k)
    ps = 16
    T, Hq = len(w.kv_len), w.cfg.num_q_heads
    out = np.full((T, Hq, k), -1, dtype=np.int32)
    perms = {}
    for t in range(T):
        b = int(w.token_seq[t])
        L = int(w.kv_len[t])
        P = -(-L // ps)
        if b not in perms:
            perms[b] = rng.permutation(-(-int(w.seq_lens[b]) // ps))
        page_of_rank = perms[b][perms[b] < P]
        wts = np.arange(1, P + 1, dtype=np.float64) ** (-alpha)
        wts /= wts.sum()
        n = min(k, L)
        draw = min(P, -(-n // ps) + 2)
        for h in range(Hq):
            ranks = rng.choice(P, size=draw, replace=False, p=wts)
            toks = page_of_rank[ranks][:, None] * ps + np.arange(ps)[None, :]
            toks = toks[toks < L][:n]
            out[t, h, :n] = np.sort(toks).astype(np.int32)
    return out


# --------------------------------------------------------------------------
# Device materialisation (bulk K/V filled on the GPU by the same definition)
# --------------------------------------------------------------------------
_FILL_LIB = None


def _fill_lib():
    global _FILL_LIB
    if _FILL_LIB is None:
        here = os.path.dirname(os.path.abspath(__file__))
        path = os.path.join(here, "libtsd_workload.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.tsdw_fill_kv.restype = ctypes.c_int
        lib.tsdw_fill_kv.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p]
        _FILL_LIB = lib
    return _FILL_LIB


@dataclass
class DeviceWorkload:
    """Device tensors of one workload, in the library's cache layout."""
    host: HostWorkload
    k: "object"            # torch uint16/bf16 [num_pages, Hkv, page_size, 128]
    v: "object"
    q: "object"            # torch bf16 [T, Hq, 128]
    page_table: "object"   # torch int32 [B, max_pages_per_seq]
    seq_lens: "object"     # torch int32 [B]
    q_indptr: "object"     # torch int32 [B+1]


def to_device(w: HostWorkload, device="cuda", stream=None) -> DeviceWorkload:
    """Materialise the cache on `device`: GPU Philox fill, then the planted rows."""
    import torch
    cfg = w.cfg
    dev = torch.device(device)
    shape = (w.num_pages, cfg.num_kv_heads, w.page_size, HEAD_DIM)
    poison_k = int(f32_to_bf16_bits(np.array([POISON_K], np.float32))[0])
    poison_v = int(f32_to_bf16_bits(np.array([POISON_V], np.float32))[0])
    k = torch.full(shape, poison_k if poison_k < 32768 else poison_k - 65536, dtype=torch.int16, device=dev)
    v = torch.full(shape, poison_v if poison_v < 32768 else poison_v - 65536, dtype=torch.int16, device=dev)
    table = torch.from_numpy(normal_table().view(np.int16)).to(dev)
    page_table = torch.from_numpy(w.page_table).to(dev)
    seq_lens = torch.from_numpy(w.seq_lens).to(dev)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    lib = _fill_lib()
    for tensor, tid in ((k, TENSOR_K), (v, TENSOR_V)):
        rc = lib.tsdw_fill_kv(tensor.data_ptr(), table.data_ptr(), page_table.data_ptr(),
                              seq_lens.data_ptr(), cfg.batch, cfg.num_kv_heads,
                              0 if cfg.layout == "contiguous" else w.page_size,
                              w.max_pages_per_seq, cfg.max_seq_len,
                              w.seed & 0xFFFFFFFF, w.seed >> 32, tid, ctypes.c_void_p(s.cuda_stream))
        if rc != 0:
            raise RuntimeError(f"workload fill failed with CUDA error {rc}")
    if w.planted_k:
        rows, vals = [], []
        for (b, g), (pos, bits) in w.planted_k.items():
            for p, r in zip(pos, bits):
                rows.append(w.physical_row(b, g, int(p)))
                vals.append(r)
        rows_t = torch.tensor(rows, dtype=torch.int64, device=dev)
        vals_t = torch.from_numpy(np.stack(vals).view(np.int16)).to(dev)
        k.view(-1, HEAD_DIM).index_copy_(0, rows_t, vals_t)
    q = torch.from_numpy(w.q_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    return DeviceWorkload(host=w, k=k.view(torch.bfloat16), v=v.view(torch.bfloat16), q=q,
                          page_table=page_table, seq_lens=seq_lens,
                          q_indptr=torch.from_numpy(w.q_indptr).to(dev))
