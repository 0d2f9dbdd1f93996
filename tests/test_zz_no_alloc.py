"""tsd_sparse_decode_static_ws: sparse decode for callers that cannot allocate.

Callers such as a plugin inside another runtime that owns all device memory,
or a decode loop that must not call cudaMalloc, get an entry point whose
scratch lives in a fixed array inside the library.  This test calls it through
the C ABI twice in a row and checks both results against tsd_sparse_decode
(which takes a caller-allocated workspace), within the parity tolerance.  The
file is named so that pytest collects it last.
"""

import ctypes
import math

import numpy as np
import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import workload as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

CFG = W.DecodeConfig(name="noalloc", batch=4, num_q_heads=16, num_kv_heads=4, seq_len=5000, ks=(120,),
                     planted=True, causal=True)


def _setup():
    import torch
    w = W.make_workload(CFG, seed=9, seq_lens=[5000, 777, 4096, 2300])
    dw = W.to_device(w, "cuda")
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=CFG.max_seq_len, page_table=dw.page_table)
    queries = tsd.Queries(dw.q, sm_scale=1.0 / math.sqrt(128))
    idx = torch.from_numpy(W.uniform_indices(w, 120)).cuda()
    return w, cache, queries, idx


def _static_call(lib, cache, queries, idx, out, lse, status, stream):
    cs, qs = cache.c_struct(), queries.c_struct()
    return lib.tsd_sparse_decode_static_ws(ctypes.byref(cs), ctypes.byref(qs), idx.data_ptr(), int(idx.shape[2]),
                                           out.data_ptr(), tsd.TSD_BF16, lse.data_ptr(), status.data_ptr(),
                                           ctypes.c_void_p(stream.cuda_stream))


def test_static_ws_matches_workspace_entry_point():
    import torch
    lib = tsd.load_library()
    w, cache, queries, idx = _setup()
    ref_out, ref_lse = tsd.sparse_decode(cache, queries, idx)
    torch.cuda.synchronize()
    ref = PT.bf16_to_np(ref_out)
    ref_l = ref_lse.cpu().numpy()
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = _static_call(lib, cache, queries, idx, out, lse, status, stream)
        assert rc == tsd.TSD_OK, tsd.status_string(rc)
        torch.cuda.synchronize()
        got = PT.bf16_to_np(out)
        allowed = PT.BF16_MAX_ABS + PT.bf16_half_ulp(ref)
        assert np.all(np.abs(got - ref) <= allowed), f"call {call}: output differs"
        assert np.allclose(lse.cpu().numpy(), ref_l, atol=PT.LSE_ABS, rtol=0), f"call {call}: lse differs"
        assert int(status.item()) == 0


def test_static_ws_rejects_shapes_beyond_its_size():
    """A shape whose scratch exceeds the array is refused before anything is launched.

    The descriptors hold placeholder addresses, so the entry point must not launch: the
    test first checks through the sizing function (host only) that the shape needs far
    more than 16 MiB, and calls the entry point only then."""
    lib = tsd.load_library()
    c = tsd._KvCacheC()
    c.k, c.v = 0x7F0000000000, 0x7F0000100000
    c.layout, c.num_kv_heads, c.head_dim, c.page_size = 0, 8, 128, 16
    c.page_table, c.max_pages_per_seq, c.num_pages = 0x7F0000200000, 8192, 512 * 8192
    c.seq_lens, c.batch, c.max_seq_len = 0x7F0000300000, 512, 131072
    q = tsd._QueriesC()
    q.q, q.q_dtype, q.num_q_heads, q.num_tokens = 0x7F0000400000, 0, 32, 2048
    q.q_indptr, q.max_tokens_per_seq, q.causal, q.sm_scale = 0x7F0000500000, 4, 1, 0.088
    need = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 2622)
    # 2048 tokens x 32 heads of split-K rows alone are 34 MB; refuse to call otherwise
    assert need > 2 * (16 << 20), f"shape no longer exceeds the static array ({need} bytes): not calling"
    rc = lib.tsd_sparse_decode_static_ws(ctypes.byref(c), ctypes.byref(q), 0x7F0000600000, 2622, 0x7F0000700000,
                                         tsd.TSD_BF16, None, None, None)
    assert rc == tsd.TSD_ERR_WORKSPACE_TOO_SMALL
