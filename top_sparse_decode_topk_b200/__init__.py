"""B200-native context-sparse decode attention: exact top-k indexer + sparse decode.

Thin Python binding over the C ABI of ``libtsd.so`` (include/tsd.h).  Every
step of the attention path runs in the library's CUDA kernels; this module only
marshals arguments (torch tensors -> device pointers, shapes, the stream) and
moves host tensors to and from the device when a caller passes them.  PyTorch
supplies device memory and streams.

The operations follow "Inference Time Context Sparsity: Illusion or
Opportunity?" (gist.science technical summary, section 2 "Oracle Top-K" and
"Hardware implementation", section 3.C):

    idx, count = topk_select(cache, queries, k_max)     # exact top-k per (token, head)
    out, lse   = sparse_decode(cache, queries, idx)      # attention over the kept rows
    out, lse   = dense_decode(cache, queries)            # attention over every row

There is no fallback: if ``libtsd.so`` is missing or a call fails, an
exception is raised.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Tuple

__all__ = [
    "KVCache", "Queries", "Workspace", "TsdError", "topk_select", "sparse_decode", "dense_decode",
    "LabelIndex", "label_channels", "label_cache_build", "topk_select_label", "stochastic_select",
    "read_device_status", "library_path", "load_library", "DEV_BAD_INDEX", "DEV_UNSORTED",
    "DEV_BAD_PAGE", "DEV_BAD_SEQ",
]

_PKG = os.path.dirname(os.path.abspath(__file__))

TSD_OK, TSD_ERR_INVALID_ARGUMENT, TSD_ERR_UNSUPPORTED = 0, 1, 2
TSD_ERR_WORKSPACE_TOO_SMALL, TSD_ERR_CUDA, TSD_ERR_DEVICE_STATUS = 3, 4, 5
TSD_BF16, TSD_F32 = 0, 1
LAYOUT_PAGED, LAYOUT_CONTIGUOUS = 0, 1
DEV_BAD_INDEX, DEV_UNSORTED, DEV_BAD_PAGE, DEV_BAD_SEQ = 1, 2, 4, 8


class TsdError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class _KvCacheC(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("layout", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("page_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages", ctypes.c_int64), ("seq_lens", ctypes.c_void_p), ("batch", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
    ]


class _QueriesC(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_dtype", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_tokens", ctypes.c_int32), ("q_indptr", ctypes.c_void_p),
        ("max_tokens_per_seq", ctypes.c_int32), ("causal", ctypes.c_int32), ("sm_scale", ctypes.c_float),
    ]


EXPORTS = {
    "tsd_version": (ctypes.c_int32, []),
    "tsd_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tsd_workspace_init": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_topk_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32]),
    "tsd_topk_select": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_sparse_decode_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC),
                                                           ctypes.c_int32]),
    "tsd_sparse_decode": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_void_p,
                                         ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_sparse_decode_host_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC),
                                                                ctypes.c_int32, ctypes.c_int32]),
    "tsd_sparse_decode_host": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_void_p,
                                              ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_dense_decode_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC)]),
    "tsd_dense_decode": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_void_p,
                                        ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "tsd_read_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "tsd_topk_select_plan": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                            ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
    "tsd_sparse_decode_plan": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                              ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                              ctypes.POINTER(ctypes.c_int32)]),
    "tsd_decode_step_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC),
                                                         ctypes.c_int32]),
    "tsd_decode_step": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "tsd_sparse_decode_static_ws": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC),
                                                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tsd_sparse_decode_weighted": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC),
                                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                                  ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                  ctypes.c_void_p]),
    "tsd_stochastic_select": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_void_p,
                                             ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tsd_topk_select_scores": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_cp_merge_select": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "tsd_merge_partials": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "tsd_label_cache_bytes": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.c_int32]),
    "tsd_label_channels_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC)]),
    "tsd_label_channels": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tsd_label_cache_build": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.c_void_p, ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tsd_topk_select_label": (ctypes.c_int, [ctypes.POINTER(_KvCacheC), ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_int32, ctypes.POINTER(_QueriesC), ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_size_t, ctypes.c_void_p]),
}

_LIB = None


def library_path() -> str:
    return os.path.join(_PKG, "libtsd.so")


def load_library():
    """Load libtsd.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing; build it with `python -m top_sparse_decode_topk_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def status_string(s: int) -> str:
    return load_library().tsd_status_string(int(s)).decode()


def _check(status: int, what: str) -> None:
    if status != TSD_OK:
        raise TsdError(status, what)


# ---------------------------------------------------------------------------
# Descriptors
# ---------------------------------------------------------------------------
@dataclass
class KVCache:
    """A bf16 KV cache on one CUDA device.

    paged:      k, v [num_pages, num_kv_heads, page_size, 128]; page_table int32 [B, max_pages];
    contiguous: k, v [B, num_kv_heads, max_seq_len, 128]; page_table None.
    seq_lens: int32 [B] on the device; max_seq_len: host bound on every entry.
    """
    k: "object"
    v: "object"
    seq_lens: "object"
    max_seq_len: int
    page_table: "object" = None

    def __post_init__(self):
        import torch
        if self.k.dtype != torch.bfloat16 or self.v.dtype != torch.bfloat16:
            raise TypeError("k and v must be bfloat16")
        if self.k.dim() != 4 or self.k.shape != self.v.shape or self.k.shape[-1] != 128:
            raise ValueError("k and v must have the same 4-d shape with head_dim 128")
        if not (self.k.is_contiguous() and self.v.is_contiguous()):
            raise ValueError("k and v must be contiguous")
        if self.seq_lens.dtype != torch.int32 or self.seq_lens.device != self.k.device:
            raise ValueError("seq_lens must be int32 on the cache's device")
        if self.page_table is None and int(self.max_seq_len) != int(self.k.shape[2]):
            raise ValueError("contiguous cache: max_seq_len must equal k.shape[2] (the token stride)")
        if self.page_table is not None:
            if self.page_table.dtype != torch.int32 or self.page_table.dim() != 2:
                raise ValueError("page_table must be an int32 [batch, max_pages] tensor")
            self.page_table = self.page_table.contiguous()

    @property
    def device(self):
        return self.k.device

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def num_kv_heads(self) -> int:
        return int(self.k.shape[1])

    def c_struct(self) -> _KvCacheC:
        key = (self.k.data_ptr(), self.v.data_ptr(), tuple(self.k.shape), self.seq_lens.data_ptr(),
               int(self.seq_lens.shape[0]), int(self.max_seq_len),
               None if self.page_table is None else (self.page_table.data_ptr(), tuple(self.page_table.shape)))
        cached = self.__dict__.get("_c_struct")
        if cached is not None and cached[0] == key:   # the same tensors: the struct is unchanged
            return cached[1]
        c = _KvCacheC()
        c.k = self.k.data_ptr()
        c.v = self.v.data_ptr()
        c.num_kv_heads = self.num_kv_heads
        c.head_dim = int(self.k.shape[3])
        c.seq_lens = self.seq_lens.data_ptr()
        c.batch = self.batch
        c.max_seq_len = int(self.max_seq_len)
        if self.page_table is None:
            c.layout = LAYOUT_CONTIGUOUS
            c.page_size = int(self.k.shape[2])
            c.page_table = None
            c.max_pages_per_seq = 1
            c.num_pages = int(self.k.shape[0])
        else:
            c.layout = LAYOUT_PAGED
            c.page_size = int(self.k.shape[2])
            c.page_table = self.page_table.data_ptr()
            c.max_pages_per_seq = int(self.page_table.shape[1])
            c.num_pages = int(self.k.shape[0])
        self.__dict__["_c_struct"] = (key, c)
        return c


@dataclass
class Queries:
    """Decode queries q [T, Hq, 128] (bf16 or fp32).

    q_indptr (int32 [B+1] on the device) gives the tokens of each sequence; None
    means one token per sequence.  max_tokens_per_seq bounds q_indptr's gaps.
    """
    q: "object"
    q_indptr: "object" = None
    max_tokens_per_seq: int = 1
    causal: bool = True
    sm_scale: Optional[float] = None

    def c_struct(self) -> _QueriesC:
        import torch
        if self.q.dim() != 3 or self.q.shape[-1] != 128 or not self.q.is_contiguous():
            raise ValueError("q must be a contiguous [T, Hq, 128] tensor")
        if self.q.dtype not in (torch.bfloat16, torch.float32):
            raise TypeError("q must be bfloat16 or float32")
        c = _QueriesC()
        c.q = self.q.data_ptr()
        c.q_dtype = TSD_BF16 if self.q.dtype == torch.bfloat16 else TSD_F32
        c.num_q_heads = int(self.q.shape[1])
        c.num_tokens = int(self.q.shape[0])
        c.q_indptr = None if self.q_indptr is None else self.q_indptr.data_ptr()
        c.max_tokens_per_seq = 1 if self.q_indptr is None else int(self.max_tokens_per_seq)
        c.causal = 1 if self.causal else 0
        c.sm_scale = float(self.sm_scale if self.sm_scale is not None else 1.0 / math.sqrt(128))
        return c


class Workspace:
    """Device scratch for the library calls (zero-initialised; the library keeps its
    leading region zero between calls).  Grows on demand; re-zeroed when the
    cache/query shapes change."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None
        self.key = None

    def get(self, nbytes: int, key, stream) -> "object":
        import torch
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            self.key = key
        elif key != self.key:
            _check(load_library().tsd_workspace_init(self.buf.data_ptr(), self.buf.numel(), stream), "workspace_init")
            self.key = key
        return self.buf


_DEFAULT_WS = {}


def _ws(workspace: Optional[Workspace], device) -> Workspace:
    if workspace is not None:
        return workspace
    key = str(device)
    if key not in _DEFAULT_WS:
        _DEFAULT_WS[key] = Workspace(device)
    return _DEFAULT_WS[key]


def _stream_ptr(stream, device):
    import torch
    s = torch.cuda.current_stream(device) if stream is None else stream
    return s, ctypes.c_void_p(s.cuda_stream)


def _shape_key(cache: KVCache, queries: Queries):
    return (cache.batch, cache.num_kv_heads, int(queries.q.shape[1]), int(queries.q.shape[0]),
            queries.max_tokens_per_seq if queries.q_indptr is not None else 1, int(cache.max_seq_len))


def _to_device(t, device, stream):
    """Host tensors are copied to `device` on `stream` (asynchronously from pinned memory)."""
    import torch
    if t is None or t.device == device:
        return t
    with torch.cuda.stream(stream):
        return t.to(device, non_blocking=True)


def _on_device_queries(queries: Queries, device, stream) -> Queries:
    if queries.q.device == device and (queries.q_indptr is None or queries.q_indptr.device == device):
        return queries
    return Queries(q=_to_device(queries.q, device, stream), q_indptr=_to_device(queries.q_indptr, device, stream),
                   max_tokens_per_seq=queries.max_tokens_per_seq, causal=queries.causal, sm_scale=queries.sm_scale)


# ---------------------------------------------------------------------------
# Operations
# ---------------------------------------------------------------------------
def topk_select(cache: KVCache, queries: Queries, k_max: int, k_per_token=None, out_idx=None, out_count=None,
                workspace: Optional[Workspace] = None, stream=None, with_scores: bool = False, out_scores=None):
    """Exact top-k token indices per (query token, q head): int32 [T, Hq, k_max]
    ascending, -1 padded, and the per-list counts int32 [T, Hq].  With `with_scores`, also
    the kept tokens' unscaled scores fp32 [T, Hq, k_max] (-inf in the padding), returned
    as (idx, scores, counts)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    queries = _on_device_queries(queries, dev, s)
    k_per_token = _to_device(k_per_token, dev, s)
    cs, qs = cache.c_struct(), queries.c_struct()
    T, Hq = int(queries.q.shape[0]), int(queries.q.shape[1])
    if out_idx is None:
        out_idx = torch.empty((T, Hq, k_max), dtype=torch.int32, device=dev)
    if out_count is None:
        out_count = torch.empty((T, Hq), dtype=torch.int32, device=dev)
    if k_per_token is not None and (k_per_token.dtype != torch.int32 or k_per_token.numel() != T):
        raise ValueError("k_per_token must be int32 [T]")
    nbytes = lib.tsd_topk_workspace_size(ctypes.byref(cs), ctypes.byref(qs), int(k_max))
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_topk_workspace_size")
    ws = _ws(workspace, dev).get(nbytes, _shape_key(cache, queries), sp)
    kp = None if k_per_token is None else k_per_token.data_ptr()
    if with_scores or out_scores is not None:
        if out_scores is None:
            out_scores = torch.empty((T, Hq, k_max), dtype=torch.float32, device=dev)
        _check(lib.tsd_topk_select_scores(ctypes.byref(cs), ctypes.byref(qs), int(k_max), kp, out_idx.data_ptr(),
                                          out_scores.data_ptr(), out_count.data_ptr(), ws.data_ptr(), ws.numel(),
                                          sp), "tsd_topk_select_scores")
        return out_idx, out_scores, out_count
    _check(lib.tsd_topk_select(ctypes.byref(cs), ctypes.byref(qs), int(k_max), kp, out_idx.data_ptr(),
                               out_count.data_ptr(), ws.data_ptr(), ws.numel(), sp), "tsd_topk_select")
    return out_idx, out_count


# ---------------------------------------------------------------------------
# Label-channel approximate indexer (Double-Sparsity-style)
# ---------------------------------------------------------------------------
@dataclass
class LabelIndex:
    """Label channels int32 [Hkv, r] and the label cache (bf16, r values per K row)."""
    channels: "object"
    label_k: "object"
    r: int


def label_channels(cache: KVCache, queries: Queries, r: int = 16, out=None, stream=None):
    """Offline choice of r label channels per kv head (int32 [Hkv, r], ascending)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    queries = _on_device_queries(queries, dev, s)
    cs, qs = cache.c_struct(), queries.c_struct()
    if out is None:
        out = torch.empty((cache.num_kv_heads, r), dtype=torch.int32, device=dev)
    nbytes = lib.tsd_label_channels_workspace_size(ctypes.byref(cs), ctypes.byref(qs))
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_label_channels_workspace_size")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib.tsd_label_channels(ctypes.byref(cs), ctypes.byref(qs), int(r), out.data_ptr(), ws.data_ptr(),
                                  ws.numel(), sp), "tsd_label_channels")
    return out


def label_cache_build(cache: KVCache, channels, status=None, stream=None) -> LabelIndex:
    """The compact label cache for `channels` (int32 [Hkv, r] on the cache's device)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    r = int(channels.shape[1])
    cs = cache.c_struct()
    nbytes = lib.tsd_label_cache_bytes(ctypes.byref(cs), r)
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_label_cache_bytes")
    label = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev)
    channels = channels.to(dev).to(torch.int32).contiguous()
    _check(lib.tsd_label_cache_build(ctypes.byref(cs), channels.data_ptr(), r, label.data_ptr(),
                                     None if status is None else status.data_ptr(), sp), "tsd_label_cache_build")
    return LabelIndex(channels=channels, label_k=label, r=r)


def topk_select_label(cache: KVCache, index: LabelIndex, queries: Queries, k_max: int, k_per_token=None,
                      out_idx=None, out_count=None, workspace: Optional[Workspace] = None, stream=None):
    """Approximate top-k over the label channels: int32 [T, Hq, k_max] ascending, -1 padded, and counts."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    queries = _on_device_queries(queries, dev, s)
    k_per_token = _to_device(k_per_token, dev, s)
    cs, qs = cache.c_struct(), queries.c_struct()
    T, Hq = int(queries.q.shape[0]), int(queries.q.shape[1])
    if out_idx is None:
        out_idx = torch.empty((T, Hq, k_max), dtype=torch.int32, device=dev)
    if out_count is None:
        out_count = torch.empty((T, Hq), dtype=torch.int32, device=dev)
    nbytes = lib.tsd_topk_workspace_size(ctypes.byref(cs), ctypes.byref(qs), int(k_max))
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_topk_workspace_size")
    ws = _ws(workspace, dev).get(nbytes, _shape_key(cache, queries), sp)
    _check(lib.tsd_topk_select_label(ctypes.byref(cs), index.label_k.data_ptr(), index.channels.data_ptr(),
                                     int(index.r), ctypes.byref(qs), int(k_max),
                                     None if k_per_token is None else k_per_token.data_ptr(),
                                     out_idx.data_ptr(), out_count.data_ptr(), ws.data_ptr(), ws.numel(), sp),
           "tsd_topk_select_label")
    return out_idx, out_count


def _out_buffers(queries, out, out_dtype, lse, dev):
    import torch
    T, Hq = int(queries.q.shape[0]), int(queries.q.shape[1])
    host_out = None
    if out is not None and out.device != dev:
        host_out = out
        out = None
    if out is None:
        out = torch.empty((T, Hq, 128), dtype=out_dtype, device=dev)
    if out.dtype not in (torch.bfloat16, torch.float32) or not out.is_contiguous():
        raise TypeError("out must be a contiguous bfloat16 or float32 tensor")
    host_lse = None
    if lse is True:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    elif lse is not None and lse is not False and lse.device != dev:
        host_lse = lse
        lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    return out, host_out, lse, host_lse


def _finish(out, host_out, lse, host_lse, stream):
    import torch
    with torch.cuda.stream(stream):
        if host_out is not None:
            host_out.copy_(out, non_blocking=True)
            out = host_out
        if host_lse is not None:
            host_lse.copy_(lse, non_blocking=True)
            lse = host_lse
    return out, lse


def sparse_decode(cache: KVCache, queries: Queries, idx, out=None, out_dtype=None, lse=True,
                  workspace: Optional[Workspace] = None, stream=None, logw=None):
    """Attention of each (token, head) over the rows of its index list.

    idx: int32 [T, Hq, k_max], each list non-decreasing then -1 padded (as
    topk_select writes it).  logw: optional fp32 [T, Hq, k_max] natural-log weight of
    each entry (tsd_sparse_decode_weighted; as stochastic_select writes it).
    Returns (out [T, Hq, 128], lse [T, Hq] or None).
    Host (CPU) inputs are copied in and a host `out`/`lse` is filled on return
    (asynchronously from/to pinned memory, ordered on `stream`).
    """
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    host = lambda x: x is not None and x is not True and x is not False and x.device.type == "cpu"
    if logw is None and host(queries.q) and host(idx) and host(out) and (lse is None or lse is False or host(lse)):
        return _sparse_decode_host(lib, cache, queries, idx, out, None if lse is False else lse, workspace, s, sp)
    queries = _on_device_queries(queries, dev, s)
    idx = _to_device(idx, dev, s)
    if idx.dtype != torch.int32 or idx.dim() != 3 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 [T, Hq, k_max] tensor")
    out_dtype = out_dtype or (out.dtype if out is not None else torch.bfloat16)
    out, host_out, lse, host_lse = _out_buffers(queries, out, out_dtype, lse, dev)
    cs, qs = cache.c_struct(), queries.c_struct()
    k_max = int(idx.shape[2])
    nbytes = lib.tsd_sparse_decode_workspace_size(ctypes.byref(cs), ctypes.byref(qs), k_max)
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_sparse_decode_workspace_size")
    ws = _ws(workspace, dev).get(nbytes, _shape_key(cache, queries), sp)
    odt = TSD_BF16 if out.dtype == torch.bfloat16 else TSD_F32
    lp = None if lse is None else lse.data_ptr()
    if logw is None:
        _check(lib.tsd_sparse_decode(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), k_max, out.data_ptr(), odt,
                                     lp, ws.data_ptr(), ws.numel(), sp), "tsd_sparse_decode")
    else:
        logw = _to_device(logw, dev, s)
        if logw.dtype != torch.float32 or tuple(logw.shape) != tuple(idx.shape) or not logw.is_contiguous():
            raise ValueError("logw must be a contiguous float32 tensor shaped like idx")
        _check(lib.tsd_sparse_decode_weighted(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), logw.data_ptr(),
                                              k_max, out.data_ptr(), odt, lp, ws.data_ptr(), ws.numel(), sp),
               "tsd_sparse_decode_weighted")
    return _finish(out, host_out, lse, host_lse, s)


def topk_select_plan(cache: KVCache, queries: Queries, k_max: int) -> dict:
    """The form topk_select would take (tsd_topk_select_plan): whether the candidate filter
    runs, and how many kernels one call launches."""
    lib = load_library()
    cs, qs = cache.c_struct(), queries.c_struct()
    f, n = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.tsd_topk_select_plan(ctypes.byref(cs), ctypes.byref(qs), int(k_max), ctypes.byref(f), ctypes.byref(n)),
           "tsd_topk_select_plan")
    return {"filtered": bool(f.value), "kernels": int(n.value)}


def sparse_decode_plan(cache: KVCache, queries: Queries, k_max: int) -> dict:
    """The work decomposition sparse_decode would use (tsd_sparse_decode_plan): the kernel's
    name, entries per task and tasks (split-K partials) per list."""
    lib = load_library()
    cs, qs = cache.c_struct(), queries.c_struct()
    p, e, c = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.tsd_sparse_decode_plan(ctypes.byref(cs), ctypes.byref(qs), int(k_max), ctypes.byref(p),
                                      ctypes.byref(e), ctypes.byref(c)), "tsd_sparse_decode_plan")
    return {"kernel": "sparse_stream_kernel" if p.value else "sparse_decode_kernel",
            "entries_per_task": e.value, "tasks_per_list": c.value}


def decode_step(cache: KVCache, queries: Queries, k_max: int, k_per_token=None, out_idx=None, out_count=None,
                out=None, out_dtype=None, lse=True, workspace: Optional[Workspace] = None, stream=None):
    """One decode step (tsd_decode_step): exact top-k, then sparse decode over the selected
    rows, on one workspace and with no host synchronisation, so that it can be captured in a
    CUDA graph.  Device tensors only.  out_idx: int32 [T, Hq, k_max] to receive the lists, or
    None to keep them in the workspace.  Returns (out, lse or None, out_idx or None)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    for name, t in (("q", queries.q), ("k_per_token", k_per_token), ("out_idx", out_idx), ("out_count", out_count),
                    ("out", out)):
        if t is not None and t.device != dev:
            raise ValueError(f"decode_step takes device tensors only ({name} is on {t.device})")
    if k_per_token is not None and (k_per_token.dtype != torch.int32 or k_per_token.numel() != queries.q.shape[0]):
        raise ValueError("k_per_token must be int32 [T]")
    out_dtype = out_dtype or (out.dtype if out is not None else torch.bfloat16)
    out, _, lse, _ = _out_buffers(queries, out, out_dtype, lse, dev)
    cs, qs = cache.c_struct(), queries.c_struct()
    nbytes = lib.tsd_decode_step_workspace_size(ctypes.byref(cs), ctypes.byref(qs), int(k_max))
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_decode_step_workspace_size")
    ws = _ws(workspace, dev).get(nbytes, _shape_key(cache, queries), sp)
    odt = TSD_BF16 if out.dtype == torch.bfloat16 else TSD_F32
    ptr = lambda t: None if t is None else t.data_ptr()
    _check(lib.tsd_decode_step(ctypes.byref(cs), ctypes.byref(qs), int(k_max), ptr(k_per_token), ptr(out_idx),
                               ptr(out_count), out.data_ptr(), odt, ptr(lse), ws.data_ptr(), ws.numel(), sp),
           "tsd_decode_step")
    return out, lse, out_idx


_HOST_WS_BYTES = {}


def _sparse_decode_host(lib, cache: KVCache, queries: Queries, idx, out, lse, workspace, s, sp):
    """sparse_decode with q, idx, out and lse in host memory: one tsd_sparse_decode_host call
    enqueues the copies in, the decode and the copies back on `s` (asynchronous: synchronise
    the stream before reading out/lse)."""
    import torch
    dev = cache.device
    if idx.dtype != torch.int32 or idx.dim() != 3 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 [T, Hq, k_max] tensor")
    if out.dtype not in (torch.bfloat16, torch.float32) or not out.is_contiguous():
        raise TypeError("out must be a contiguous bfloat16 or float32 tensor")
    if not queries.q.is_contiguous():
        raise ValueError("q must be contiguous")
    T, Hq = int(queries.q.shape[0]), int(queries.q.shape[1])
    if tuple(out.shape) != (T, Hq, 128) or int(idx.shape[0]) != T or int(idx.shape[1]) != Hq:
        raise ValueError("q, idx and out shapes disagree")
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (T, Hq) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [T, Hq] tensor")
    qd = queries if queries.q_indptr is None or queries.q_indptr.device == dev else Queries(
        q=queries.q, q_indptr=_to_device(queries.q_indptr, dev, s), max_tokens_per_seq=queries.max_tokens_per_seq,
        causal=queries.causal, sm_scale=queries.sm_scale)
    cs, qs = cache.c_struct(), qd.c_struct()
    k_max = int(idx.shape[2])
    odt = TSD_BF16 if out.dtype == torch.bfloat16 else TSD_F32
    skey = _shape_key(cache, qd)
    size_key = (str(dev), skey, k_max, odt, qs.q_dtype)   # the work split depends on the device's SM count
    nbytes = _HOST_WS_BYTES.get(size_key)
    if nbytes is None:   # the size depends only on the shapes: asked once per shape
        nbytes = lib.tsd_sparse_decode_host_workspace_size(ctypes.byref(cs), ctypes.byref(qs), k_max, odt)
        if nbytes == 0:
            raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_sparse_decode_host_workspace_size")
        _HOST_WS_BYTES[size_key] = nbytes
    ws = _ws(workspace, dev).get(nbytes, skey, sp)
    _check(lib.tsd_sparse_decode_host(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), k_max, out.data_ptr(), odt,
                                      None if lse is None else lse.data_ptr(), ws.data_ptr(), ws.numel(), sp),
           "tsd_sparse_decode_host")
    return out, lse


def stochastic_select(cache: KVCache, queries: Queries, topk_idx, u, status=None, stream=None):
    """vAttention-style selection: the top-k lists plus m uniform samples of the other tokens.

    topk_idx: int32 [T, Hq, k_max] (as topk_select writes it); u: uint32-valued int32 or
    int64 [T, Hq, m] random words.  Returns (idx int32 [T, Hq, k_max + m] ascending, -1
    padded; logw fp32 of the same shape: 0 for top-k entries, ln(|rest| / m') for samples)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    queries = _on_device_queries(queries, dev, s)
    topk_idx = _to_device(topk_idx, dev, s).contiguous()
    u = _to_device(u, dev, s)
    if u.dtype != torch.int32:
        u = (u.to(torch.int64) & 0xFFFFFFFF).to(torch.int64)
        u = torch.where(u >= 2**31, u - 2**32, u).to(torch.int32)   # same 32-bit words
    u = u.contiguous()
    T, Hq, k_max = (int(x) for x in topk_idx.shape)
    m = int(u.shape[2])
    idx = torch.empty((T, Hq, k_max + m), dtype=torch.int32, device=dev)
    logw = torch.empty((T, Hq, k_max + m), dtype=torch.float32, device=dev)
    cs, qs = cache.c_struct(), queries.c_struct()
    _check(lib.tsd_stochastic_select(ctypes.byref(cs), ctypes.byref(qs), topk_idx.data_ptr(), k_max, u.data_ptr(), m,
                                     idx.data_ptr(), logw.data_ptr(), None if status is None else status.data_ptr(),
                                     sp), "tsd_stochastic_select")
    return idx, logw


def dense_decode(cache: KVCache, queries: Queries, out=None, out_dtype=None, lse=True,
                 workspace: Optional[Workspace] = None, stream=None):
    """Dense decode attention over every visible token (the comparator)."""
    import torch
    lib = load_library()
    dev = cache.device
    s, sp = _stream_ptr(stream, dev)
    queries = _on_device_queries(queries, dev, s)
    out_dtype = out_dtype or (out.dtype if out is not None else torch.bfloat16)
    out, host_out, lse, host_lse = _out_buffers(queries, out, out_dtype, lse, dev)
    cs, qs = cache.c_struct(), queries.c_struct()
    nbytes = lib.tsd_dense_decode_workspace_size(ctypes.byref(cs), ctypes.byref(qs))
    if nbytes == 0:
        raise TsdError(TSD_ERR_INVALID_ARGUMENT, "tsd_dense_decode_workspace_size")
    ws = _ws(workspace, dev).get(nbytes, _shape_key(cache, queries), sp)
    _check(lib.tsd_dense_decode(ctypes.byref(cs), ctypes.byref(qs), out.data_ptr(),
                                TSD_BF16 if out.dtype == torch.bfloat16 else TSD_F32,
                                None if lse is None else lse.data_ptr(), ws.data_ptr(), ws.numel(), sp),
           "tsd_dense_decode")
    return _finish(out, host_out, lse, host_lse, s)


def read_device_status(workspace: Optional[Workspace] = None, device=None, stream=None) -> int:
    """Read and clear the device status bits of a workspace (synchronises the stream)."""
    import torch
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    ws = _ws(workspace, dev)
    if ws.buf is None:
        return 0
    s, sp = _stream_ptr(stream, ws.buf.device)
    flags = ctypes.c_uint32(0)
    rc = lib.tsd_read_device_status(ws.buf.data_ptr(), sp, ctypes.byref(flags))
    if rc not in (TSD_OK, TSD_ERR_DEVICE_STATUS):
        raise TsdError(rc, "tsd_read_device_status")
    return int(flags.value)
