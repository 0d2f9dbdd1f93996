"""Context-parallel decode over a token-sharded paged KV cache (host orchestration).

Each rank holds a token range of every sequence: rank r keeps tokens
[r * S, (r + 1) * S) with S a multiple of the page size.  A decode step on rank r:

1. exact top-k of its shard with the kept scores (``topk_select(..., with_scores=True)``);
2. gather of every rank's (local index, score) candidates, rank-major;
3. ``cp_merge_select``: the global top-k among the P x k candidates -- it is contained in the
   union of the local top-k lists -- keeping this rank's kept entries;
4. sparse decode of the shard over them, fp32 output and log-sum-exp;
5. gather of the P partial (output, lse) pairs and ``merge_partials``.

Steps 1, 3, 4 and 5 are this library's kernels; the gathers are the caller's collective
(``torch.distributed.all_gather_into_tensor`` over NCCL, see ``gather_rank_major``).  Only
single-token decode (one query per sequence) is supported: a shard's visible length is then
clamp(seq_len - r * S, 0, S) for every query.
"""

from __future__ import annotations

import ctypes
from typing import Callable, Tuple

from . import (KVCache, Queries, TsdError, TSD_BF16, TSD_F32, TSD_ERR_INVALID_ARGUMENT, _check, load_library,
               _stream_ptr, sparse_decode, topk_select)

__all__ = ["shard_length", "shard_view", "cp_merge_select", "merge_partials", "gather_rank_major", "cp_decode_step"]


def shard_length(max_seq_len: int, world: int, page_size: int) -> int:
    """Tokens per rank: ceil(max_seq_len / world) rounded up to whole pages."""
    s = -(-int(max_seq_len) // int(world))
    return -(-s // int(page_size)) * int(page_size)


def shard_view(cache: KVCache, rank: int, world: int) -> KVCache:
    """Rank `rank`'s shard of a paged cache, sharing its pages: the page-table columns of
    the rank's token range and the visible lengths clamped to it."""
    import torch
    if cache.page_table is None:
        raise ValueError("context-parallel sharding needs a paged cache")
    ps = int(cache.k.shape[2])
    S = shard_length(cache.max_seq_len, world, ps)
    begin = rank * S
    p0 = begin // ps
    pages = S // ps
    pt = cache.page_table[:, p0:p0 + pages]
    if pt.shape[1] < pages:   # last shard past the table: pad with unused (-1) columns
        pad = torch.full((pt.shape[0], pages - pt.shape[1]), -1, dtype=pt.dtype, device=pt.device)
        pt = torch.cat([pt, pad], dim=1)
    lens = torch.clamp(cache.seq_lens - begin, 0, S).to(torch.int32)
    return KVCache(cache.k, cache.v, lens, max_seq_len=S, page_table=pt.contiguous())


def cp_merge_select(cand_idx, cand_scores, k: int, my_rank: int, k_out=None, status=None, stream=None):
    """Global top-k among rank-major candidates [P, T, Hq, kc]; returns rank my_rank's kept
    local indices int32 [T, Hq, k_out] (k_out defaults to k), ascending, -1 padded."""
    import torch
    lib = load_library()
    dev = cand_idx.device
    s, sp = _stream_ptr(stream, dev)
    P, T, Hq, kc = (int(x) for x in cand_idx.shape)
    k_out = int(k if k_out is None else k_out)
    out = torch.empty((T, Hq, k_out), dtype=torch.int32, device=dev)
    _check(lib.tsd_cp_merge_select(cand_idx.contiguous().data_ptr(), cand_scores.contiguous().data_ptr(), P, T * Hq,
                                   kc, None, int(k), int(my_rank), out.data_ptr(), k_out,
                                   None if status is None else status.data_ptr(), sp), "tsd_cp_merge_select")
    return out


def merge_partials(out_parts, lse_parts, out_dtype=None, stream=None) -> Tuple["object", "object"]:
    """Merge P partial decodes: out_parts fp32 [P, T, Hq, 128], lse_parts [P, T, Hq]."""
    import torch
    lib = load_library()
    dev = out_parts.device
    s, sp = _stream_ptr(stream, dev)
    P, T, Hq, D = (int(x) for x in out_parts.shape)
    out_dtype = out_dtype or torch.bfloat16
    out = torch.empty((T, Hq, D), dtype=out_dtype, device=dev)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    _check(lib.tsd_merge_partials(P, T * Hq, out_parts.contiguous().data_ptr(), lse_parts.contiguous().data_ptr(),
                                  out.data_ptr(), TSD_F32 if out_dtype == torch.float32 else TSD_BF16,
                                  lse.data_ptr(), sp), "tsd_merge_partials")
    return out, lse


def gather_rank_major(t, group=None):
    """[P, *t.shape] of every rank's `t`, rank-major, through torch.distributed."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    t = t.contiguous()
    # concatenated along the first dimension (the form every backend accepts), then viewed
    out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t, group=group)
    return out.view((world,) + tuple(t.shape))


def cp_decode_step(shard: KVCache, queries: Queries, k: int, rank: int,
                   gather: Callable = gather_rank_major, out_dtype=None, workspace=None):
    """One single-token decode step over a token-sharded cache (see the module header)."""
    import torch
    if queries.q_indptr is not None:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "context-parallel decode supports one query per sequence")
    idx, scores, _ = topk_select(shard, queries, k, with_scores=True, workspace=workspace)
    cand_idx, cand_scores = gather(idx), gather(scores)
    mine = cp_merge_select(cand_idx, cand_scores, k, rank)
    out_r, lse_r = sparse_decode(shard, queries, mine, out_dtype=torch.float32, workspace=workspace)
    return merge_partials(gather(out_r), gather(lse_r), out_dtype=out_dtype)
