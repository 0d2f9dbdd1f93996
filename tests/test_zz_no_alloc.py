"""tsd_sparse_decode_static_ws: sparse decode for callers that cannot allocate.

Some callers have no way to obtain device memory for a workspace: a plugin running
inside another runtime that owns every device allocation, or a decode loop that must
not call cudaMalloc (it synchronizes the whole device).  For them the library offers
an entry point whose scratch is a fixed array inside the library itself.

These tests call it through the C ABI, several times in a row, and check that:
* it returns exactly (bit for bit) what tsd_sparse_decode returns with a
  caller-allocated workspace -- the plan and the kernel are the same -- and that both
  match the float64 oracle on every list;
* with no status pointer (the status word then lives in the shared array) and fp32
  output it still matches, and a larger shape after a smaller one, then the smaller
  one again, sees no stale merge counters or partials;
* a shape whose scratch exceeds the array is refused without launching.  The refused
  call gets real device buffers of the declared shapes, so that a drift between the
  sizing rule and the entry point's own check could only ever launch on valid memory.

The file is named so that pytest collects it last.
"""

import ctypes
import math

import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

SM_SCALE = 1.0 / math.sqrt(128)
STATIC_BYTES = 16 << 20   # the array's size, as include/tsd.h states it

SMALL = W.DecodeConfig(name="noalloc", batch=4, num_q_heads=16, num_kv_heads=4, seq_len=5000, ks=(120,),
                       planted=True, causal=True)
SMALL_LENS = [5000, 777, 4096, 2300]
LARGER = W.DecodeConfig(name="noalloc_larger", batch=6, num_q_heads=16, num_kv_heads=4, seq_len=6000,
                        tokens_per_seq=2, ks=(300,), planted=True, causal=True)
LARGER_LENS = [6000, 1200, 5999, 3000, 4500, 900]


def _setup(cfg, lens, seed, k):
    import torch
    w = W.make_workload(cfg, seed=seed, seq_lens=lens)
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=cfg.max_seq_len, page_table=dw.page_table)
    multi = cfg.tokens_per_seq > 1
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=cfg.causal, sm_scale=SM_SCALE)
    idx_np = W.uniform_indices(w, k)
    return w, cache, queries, idx_np, torch.from_numpy(idx_np).cuda()


def _static_call(lib, cache, queries, idx, out, out_dtype, lse, status, stream):
    cs, qs = cache.c_struct(), queries.c_struct()
    return lib.tsd_sparse_decode_static_ws(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), int(idx.shape[2]),
                                           out.data_ptr(), out_dtype, lse.data_ptr(),
                                           None if status is None else status.data_ptr(),
                                           ctypes.c_void_p(stream.cuda_stream))


def _all_pairs(w):
    return [(t, h) for t in range(len(w.kv_len)) for h in range(w.cfg.num_q_heads)]


def _check(case, calls, f32, with_status):
    """`calls` static-scratch calls on `case`: each bit-identical to the workspace entry
    point's result, and that result within the oracle's bar on every list."""
    import torch
    lib = tsd.load_library()
    w, cache, queries, idx_np, idx = case
    odt = torch.float32 if f32 else torch.bfloat16
    ref_out, ref_lse = tsd.sparse_decode(cache, queries, idx, out_dtype=odt)
    torch.cuda.synchronize()
    assert tsd.read_device_status() == 0
    PT.check_decode(PT.OracleInputs(w), idx_np, PT.bf16_to_np(ref_out), ref_lse.cpu().numpy(), _all_pairs(w),
                    SM_SCALE, out_is_bf16=not f32)
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device="cuda") if with_status else None
    for call in range(calls):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = _static_call(lib, cache, queries, idx, out, tsd.TSD_F32 if f32 else tsd.TSD_BF16, lse, status, stream)
        assert rc == tsd.TSD_OK, tsd.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), f"call {call}: output differs from the workspace entry point"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from the workspace entry point"
        if status is not None:
            assert int(status.item()) == 0


def test_static_ws_matches_workspace_entry_point():
    """bf16 output with a status word, two calls in a row."""
    _check(_setup(SMALL, SMALL_LENS, 9, 120), calls=2, f32=False, with_status=True)


def test_static_ws_larger_shape_then_smaller_again():
    """fp32 output with no status pointer on a larger, multi-token shape (more lists, more
    splits per list), then the first shape again: the array's merge counters and partials
    are re-cleared or overwritten between calls of different shapes."""
    _check(_setup(LARGER, LARGER_LENS, 4, 300), calls=2, f32=True, with_status=False)
    _check(_setup(SMALL, SMALL_LENS, 9, 120), calls=2, f32=False, with_status=False)


def test_static_ws_rejects_shapes_beyond_its_size():
    """2048 one-token sequences x 32 q heads need more than 16 MiB of split-K rows even at one
    split per list.  Every pointer handed over is a real device buffer of the declared shape
    (contiguous cache, zero-filled index lists), and the size is checked through the host-only
    sizing function before the call."""
    import torch
    lib = tsd.load_library()
    B, hq, hkv, n, k = 2048, 32, 1, 16, 16
    k_cache = torch.zeros((B, hkv, n, 128), dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    seq_lens = torch.full((B,), n, dtype=torch.int32, device="cuda")
    q = torch.zeros((B, hq, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((B, hq, k), dtype=torch.int32, device="cuda")
    out = torch.zeros((B, hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, hq), dtype=torch.float32, device="cuda")
    cache = tsd.KVCache(k_cache, v_cache, seq_lens, max_seq_len=n)
    queries = tsd.Queries(q, sm_scale=SM_SCALE)
    cs, qs = cache.c_struct(), queries.c_struct()
    need = lib.tsd_sparse_decode_workspace_size(ctypes.byref(cs), ctypes.byref(qs), k)
    assert need > STATIC_BYTES, f"shape no longer exceeds the static array ({need} bytes)"
    stream = torch.cuda.current_stream()
    out_before = out.clone()
    rc = lib.tsd_sparse_decode_static_ws(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), k, out.data_ptr(),
                                         tsd.TSD_BF16, lse.data_ptr(), None, ctypes.c_void_p(stream.cuda_stream))
    torch.cuda.synchronize()
    assert rc == tsd.TSD_ERR_WORKSPACE_TOO_SMALL, tsd.status_string(rc)
    assert torch.equal(out, out_before)   # nothing ran
