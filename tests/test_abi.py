"""The C-ABI library without a GPU: it loads, exports what include/tsd.h declares,
and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

import top_sparse_decode_topk_b200 as tsd
from top_sparse_decode_topk_b200 import _KvCacheC, _QueriesC
from top_sparse_decode_topk_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tsd.h")


def _gpu_visible() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# Calls below hand the library placeholder device addresses and expect it to refuse
# them on the host.  Where a GPU is visible they are skipped, so that a regression in a
# host check can never turn into a launch on those addresses.
fake_pointer_call = pytest.mark.skipif(_gpu_visible(), reason="placeholder-address calls run only without a GPU")


@pytest.fixture(scope="module")
def lib():
    build()
    return tsd.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tsd_[a-z_]+)\s*\(", text)))


def test_header_declares_the_path(lib):
    names = declared_functions()
    for need in ("tsd_topk_select", "tsd_sparse_decode", "tsd_dense_decode", "tsd_read_device_status"):
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # the binding declares the same set
    assert set(declared_functions()) == set(tsd.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.tsd_version() >= 100
    assert tsd.status_string(0) == "TSD_OK"
    assert tsd.status_string(3) == "TSD_ERR_WORKSPACE_TOO_SMALL"
    assert tsd.status_string(99) == "TSD_UNKNOWN_STATUS"


FAKE = 0x7F0000000000   # 256-byte aligned, never dereferenced by the host checks


def make_cache(**kw):
    c = _KvCacheC()
    c.k, c.v = FAKE, FAKE + 0x100000
    c.layout = kw.get("layout", 0)
    c.num_kv_heads = kw.get("hkv", 8)
    c.head_dim = kw.get("head_dim", 128)
    c.page_size = kw.get("page_size", 16)
    c.page_table = kw.get("page_table", FAKE + 0x200000)
    c.max_pages_per_seq = kw.get("max_pages", 2048)
    c.num_pages = kw.get("num_pages", 8 * 2048)
    c.seq_lens = FAKE + 0x300000
    c.batch = kw.get("batch", 8)
    c.max_seq_len = kw.get("max_seq_len", 32768)
    return c


def make_queries(**kw):
    q = _QueriesC()
    q.q = kw.get("q", FAKE + 0x400000)
    q.q_dtype = kw.get("q_dtype", 0)
    q.num_q_heads = kw.get("hq", 32)
    q.num_tokens = kw.get("tokens", 8)
    q.q_indptr = kw.get("q_indptr", None)
    q.max_tokens_per_seq = kw.get("max_tokens", 1)
    q.causal = 1
    q.sm_scale = kw.get("sm_scale", 0.088)
    return q


def sparse(lib, c, q, k_max=655, ws_bytes=1 << 40, out_dtype=0, idx=FAKE + 0x500000):
    return lib.tsd_sparse_decode(ctypes.byref(c), ctypes.byref(q), idx, k_max, FAKE + 0x600000, out_dtype,
                                 None, FAKE + 0x700000, ws_bytes, None)


def test_workspace_sizes(lib):
    c, q = make_cache(), make_queries()
    s1 = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    s2 = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 13107)
    d = lib.tsd_dense_decode_workspace_size(ctypes.byref(c), ctypes.byref(q))
    t = lib.tsd_topk_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    assert 0 < s1 <= s2 and d > 0
    # top-k holds one fp32 score per (token, head, position)
    assert t >= 8 * 32 * 32768 * 4
    bad = make_cache(head_dim=64)
    assert lib.tsd_sparse_decode_workspace_size(ctypes.byref(bad), ctypes.byref(q), 655) == 0
    assert lib.tsd_topk_workspace_size(ctypes.byref(c), ctypes.byref(q), 0) == 0


@fake_pointer_call
@pytest.mark.parametrize("mutate,status", [
    (dict(head_dim=64), tsd.TSD_ERR_UNSUPPORTED),
    (dict(page_size=24), tsd.TSD_ERR_UNSUPPORTED),
    (dict(hkv=5), tsd.TSD_ERR_INVALID_ARGUMENT),        # 32 % 5 != 0
    (dict(batch=0), tsd.TSD_ERR_INVALID_ARGUMENT),
    (dict(max_pages=10), tsd.TSD_ERR_INVALID_ARGUMENT),  # 10 * 16 < max_seq_len
    (dict(layout=7), tsd.TSD_ERR_INVALID_ARGUMENT),
    (dict(page_table=None), tsd.TSD_ERR_INVALID_ARGUMENT),
])
def test_cache_errors_before_launch(lib, mutate, status):
    assert sparse(lib, make_cache(**mutate), make_queries()) == status


@fake_pointer_call
@pytest.mark.parametrize("mutate,status", [
    (dict(tokens=7), tsd.TSD_ERR_INVALID_ARGUMENT),      # no q_indptr: T must equal batch
    (dict(q_dtype=9), tsd.TSD_ERR_UNSUPPORTED),
    (dict(sm_scale=0.0), tsd.TSD_ERR_INVALID_ARGUMENT),
    (dict(q=FAKE + 8), tsd.TSD_ERR_INVALID_ARGUMENT),    # misaligned rows
    (dict(q=None), tsd.TSD_ERR_INVALID_ARGUMENT),
])
def test_query_errors_before_launch(lib, mutate, status):
    assert sparse(lib, make_cache(), make_queries(**mutate)) == status


@fake_pointer_call
def test_other_errors_before_launch(lib):
    c, q = make_cache(), make_queries()
    assert sparse(lib, c, q, ws_bytes=1024) == tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert sparse(lib, c, q, k_max=0) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert sparse(lib, c, q, idx=None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert sparse(lib, c, q, out_dtype=5) == tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_sparse_decode(None, ctypes.byref(q), FAKE, 8, FAKE, 0, None, FAKE, 1 << 40, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_dense_decode(ctypes.byref(c), ctypes.byref(q), FAKE, 0, None, FAKE, 16, None) == \
        tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert lib.tsd_topk_select(ctypes.byref(c), ctypes.byref(q), 655, None, FAKE, None, FAKE, 16, None) == \
        tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert lib.tsd_topk_select(ctypes.byref(c), ctypes.byref(q), 655, None, None, None, FAKE, 1 << 40, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT
    flags = ctypes.c_uint32(0)
    assert lib.tsd_read_device_status(None, None, ctypes.byref(flags)) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_workspace_init(None, 0, None) == tsd.TSD_OK
    assert lib.tsd_workspace_init(None, 16, None) == tsd.TSD_ERR_INVALID_ARGUMENT


@fake_pointer_call
def test_host_buffer_decode_errors_before_any_copy(lib):
    """tsd_sparse_decode_host rejects what tsd_sparse_decode rejects, before it enqueues a copy."""
    c, q = make_cache(), make_queries()
    sz = lib.tsd_sparse_decode_host_workspace_size(ctypes.byref(c), ctypes.byref(q), 655, 0)
    base = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    # the decode workspace, then staging for q (bf16), the lists, out (bf16) and lse
    assert sz >= base + 8 * 32 * (128 * 2 + 655 * 4 + 128 * 2 + 4)
    assert lib.tsd_sparse_decode_host_workspace_size(ctypes.byref(c), ctypes.byref(q), 655, 5) == 0
    assert lib.tsd_sparse_decode_host_workspace_size(ctypes.byref(c), ctypes.byref(q), 0, 0) == 0

    def host(cc=c, qq=q, k_max=655, out_dtype=0, idx=FAKE + 0x500000, ws_bytes=1 << 40):
        return lib.tsd_sparse_decode_host(ctypes.byref(cc), ctypes.byref(qq), idx, k_max, FAKE + 0x600000, out_dtype,
                                          None, FAKE + 0x700000, ws_bytes, None)
    assert host(ws_bytes=base) == tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert host(k_max=0) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert host(idx=None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert host(out_dtype=5) == tsd.TSD_ERR_UNSUPPORTED
    assert host(cc=make_cache(head_dim=64)) == tsd.TSD_ERR_UNSUPPORTED
    assert host(qq=make_queries(sm_scale=0.0)) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_sparse_decode_host(None, ctypes.byref(q), FAKE, 8, FAKE, 0, None, FAKE, 1 << 40, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT


@fake_pointer_call
def test_multi_token_queries_need_bounds(lib):
    c = make_cache(batch=32)
    q = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=0)
    assert sparse(lib, c, q) == tsd.TSD_ERR_INVALID_ARGUMENT
    q = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=4)
    assert lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 2622) > 0


@fake_pointer_call
def test_label_and_stochastic_errors_before_launch(lib):
    c, q = make_cache(), make_queries()
    # label cache sizing is host arithmetic: rows x r x 2 bytes, 0 for an unsupported r
    rows = c.num_pages * c.num_kv_heads * c.page_size
    assert lib.tsd_label_cache_bytes(ctypes.byref(c), 16) == rows * 16 * 2
    assert lib.tsd_label_cache_bytes(ctypes.byref(c), 12) == 0
    assert lib.tsd_label_channels_workspace_size(ctypes.byref(c), ctypes.byref(q)) > 256
    assert lib.tsd_label_channels(ctypes.byref(c), ctypes.byref(q), 12, FAKE, FAKE, 1 << 30, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_label_channels(ctypes.byref(c), ctypes.byref(q), 16, FAKE, FAKE, 16, None) == \
        tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert lib.tsd_label_cache_build(ctypes.byref(c), FAKE, 24, FAKE, None, None) == tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_label_cache_build(ctypes.byref(c), None, 16, FAKE, None, None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_label_cache_build(ctypes.byref(c), FAKE, 16, FAKE + 8, None, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT   # misaligned label cache
    assert lib.tsd_topk_select_label(ctypes.byref(c), FAKE, FAKE, 16, ctypes.byref(q), 655, None, FAKE, None,
                                     FAKE, 16, None) == tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    assert lib.tsd_topk_select_label(ctypes.byref(c), FAKE, FAKE, 20, ctypes.byref(q), 655, None, FAKE, None,
                                     FAKE, 1 << 40, None) == tsd.TSD_ERR_UNSUPPORTED
    # stochastic selection and weighted decode
    assert lib.tsd_stochastic_select(ctypes.byref(c), ctypes.byref(q), FAKE, 655, FAKE, 2048, FAKE, FAKE, None,
                                     None) == tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_stochastic_select(ctypes.byref(c), ctypes.byref(q), FAKE, 655, None, 64, FAKE, FAKE, None,
                                     None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_stochastic_select(ctypes.byref(c), ctypes.byref(q), None, 655, FAKE, 64, FAKE, FAKE, None,
                                     None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_sparse_decode_weighted(ctypes.byref(c), ctypes.byref(q), FAKE, None, 655, FAKE, 0, None, FAKE,
                                          1 << 40, None) == tsd.TSD_ERR_INVALID_ARGUMENT


@fake_pointer_call
def test_context_parallel_errors_before_launch(lib):
    c, q = make_cache(), make_queries()
    assert lib.tsd_topk_select_scores(ctypes.byref(c), ctypes.byref(q), 655, None, FAKE, None, None, FAKE, 1 << 40,
                                      None) == tsd.TSD_ERR_INVALID_ARGUMENT      # no score buffer
    # ranks x candidates above what one CTA holds
    assert lib.tsd_cp_merge_select(FAKE, FAKE, 8, 256, 4096, None, 655, 0, FAKE, 655, None, None) == \
        tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_cp_merge_select(FAKE, FAKE, 4, 256, 655, None, 655, 4, FAKE, 655, None, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT   # my_rank outside [0, ranks)
    assert lib.tsd_cp_merge_select(None, FAKE, 4, 256, 655, None, 655, 0, FAKE, 655, None, None) == \
        tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_merge_partials(4, 256, FAKE, FAKE, FAKE, 7, None, None) == tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_merge_partials(0, 256, FAKE, FAKE, FAKE, 0, None, None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_merge_partials(4, 256, FAKE + 4, FAKE, FAKE, 0, None, None) == tsd.TSD_ERR_INVALID_ARGUMENT


@fake_pointer_call
def test_static_scratch_refuses_oversize_shapes(lib):
    """tsd_sparse_decode_static_ws refuses, on the host, a shape whose scratch exceeds its
    16 MiB array: 2048 tokens x 32 heads of split-K rows alone are over 34 MB."""
    c = make_cache(batch=512, max_pages=8192, num_pages=512 * 8192, max_seq_len=131072)
    q = make_queries(tokens=2048, q_indptr=FAKE + 0x800000, max_tokens=4)
    need = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 2622)
    assert need > 2 * (16 << 20)
    rc = lib.tsd_sparse_decode_static_ws(ctypes.byref(c), ctypes.byref(q), FAKE + 0x500000, 2622, FAKE + 0x600000,
                                         tsd.TSD_BF16, None, None, None)
    assert rc == tsd.TSD_ERR_WORKSPACE_TOO_SMALL
    # and rejects bad arguments the way tsd_sparse_decode does
    assert lib.tsd_sparse_decode_static_ws(ctypes.byref(make_cache(head_dim=64)), ctypes.byref(make_queries()),
                                           FAKE, 8, FAKE, 0, None, None, None) == tsd.TSD_ERR_UNSUPPORTED
    assert lib.tsd_sparse_decode_static_ws(ctypes.byref(make_cache()), ctypes.byref(make_queries()), None, 8, FAKE,
                                           0, None, None, None) == tsd.TSD_ERR_INVALID_ARGUMENT


@fake_pointer_call
def test_decode_step_errors_before_launch(lib):
    """tsd_decode_step checks what both of its calls check before it enqueues anything, and
    sizes one region for the two workspaces (plus the lists when the caller keeps none)."""
    c, q = make_cache(), make_queries()
    step = lib.tsd_decode_step_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    topk = lib.tsd_topk_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    dec = lib.tsd_sparse_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    assert step >= max(topk, dec) + 8 * 32 * 655 * 4
    assert step < topk + dec + 8 * 32 * 655 * 4 + 1024   # one shared region, not two
    assert lib.tsd_decode_step_workspace_size(ctypes.byref(c), ctypes.byref(q), 0) == 0

    def call(cc=c, qq=q, k_max=655, out=FAKE + 0x600000, out_dtype=0, ws=FAKE + 0x700000, ws_bytes=1 << 40,
             out_idx=None):
        return lib.tsd_decode_step(ctypes.byref(cc), ctypes.byref(qq), k_max, None, out_idx, None, out, out_dtype,
                                   None, ws, ws_bytes, None)
    assert call(ws_bytes=max(topk, dec)) == tsd.TSD_ERR_WORKSPACE_TOO_SMALL   # no room for the lists
    assert call(k_max=0) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert call(out=None) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert call(out_dtype=5) == tsd.TSD_ERR_UNSUPPORTED
    assert call(ws=FAKE + 0x700010) == tsd.TSD_ERR_INVALID_ARGUMENT        # workspace not 256-byte aligned
    assert call(cc=make_cache(head_dim=64)) == tsd.TSD_ERR_UNSUPPORTED
    assert call(k_max=1 << 20) == tsd.TSD_ERR_UNSUPPORTED


def test_sparse_decode_plan_choice(lib):
    """The work decomposition query (host arithmetic only).  One decode token per sequence and
    k = 655 over 8 sequences x 8 kv heads x 4 q heads fits one wave as 4 chunks of 176 entries;
    the ragged shape (128 tokens, 32 heads, k up to 2622) needs more than one wave and takes the
    persistent kernel with 512-entry chunks (148 SMs assumed without a device)."""
    c, q = make_cache(), make_queries()
    p, e, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    args = (ctypes.byref(p), ctypes.byref(e), ctypes.byref(n))
    try:
        import torch
        if torch.cuda.is_available() and torch.cuda.get_device_properties(0).multi_processor_count != 148:
            pytest.skip("the expected splits assume 148 SMs")
    except ImportError:
        pass
    assert lib.tsd_sparse_decode_plan(ctypes.byref(c), ctypes.byref(q), 655, *args) == tsd.TSD_OK
    assert (p.value, e.value, n.value) == (0, 176, 4)
    rc = make_cache(batch=32, max_pages=8192, num_pages=32 * 8192, max_seq_len=131072)
    rq = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=4)
    assert lib.tsd_sparse_decode_plan(ctypes.byref(rc), ctypes.byref(rq), 2622, *args) == tsd.TSD_OK
    assert (p.value, e.value, n.value) == (1, 512, 6)
    assert lib.tsd_sparse_decode_plan(ctypes.byref(c), ctypes.byref(q), 0, *args) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_sparse_decode_plan(ctypes.byref(c), ctypes.byref(q), 655, None, ctypes.byref(e),
                                      ctypes.byref(n)) == tsd.TSD_ERR_INVALID_ARGUMENT
    bad = make_cache(head_dim=64)
    assert lib.tsd_sparse_decode_plan(ctypes.byref(bad), ctypes.byref(q), 655, *args) == tsd.TSD_ERR_UNSUPPORTED


def test_topk_select_plan_choice(lib, monkeypatch):
    """Which form of the exact indexer a call takes (host arithmetic only).  The Llama-3-8B shape
    (256 lists x 32K tokens: 33.5 MB of score rows, which stay in L2) takes the form over score
    rows, 2 kernels; the ragged shape (4096 lists x 128K: 2.1 GB of rows) the candidate filter, 4
    kernels; fp32 queries, a k too large for the candidate buffer and TSD_TOPK_FILTER=0 all give
    the row form, and TSD_TOPK_FILTER=1 forces the filter on the small shape."""
    monkeypatch.delenv("TSD_TOPK_FILTER", raising=False)
    monkeypatch.delenv("TSD_SCORE_KERNEL", raising=False)
    f, n = ctypes.c_int32(), ctypes.c_int32()
    args = (ctypes.byref(f), ctypes.byref(n))
    c, q = make_cache(), make_queries()
    assert lib.tsd_topk_select_plan(ctypes.byref(c), ctypes.byref(q), 655, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (0, 2)
    rc = make_cache(batch=32, max_pages=8192, num_pages=32 * 8192, max_seq_len=131072)
    rq = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=4)
    assert lib.tsd_topk_select_plan(ctypes.byref(rc), ctypes.byref(rq), 2622, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (1, 4)
    rq32 = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=4, q_dtype=tsd.TSD_F32)
    assert lib.tsd_topk_select_plan(ctypes.byref(rc), ctypes.byref(rq32), 2622, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (0, 2)
    assert lib.tsd_topk_select_plan(ctypes.byref(rc), ctypes.byref(rq), 13107, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (0, 2)
    monkeypatch.setenv("TSD_TOPK_FILTER", "0")
    assert lib.tsd_topk_select_plan(ctypes.byref(rc), ctypes.byref(rq), 2622, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (0, 2)
    monkeypatch.setenv("TSD_TOPK_FILTER", "1")
    assert lib.tsd_topk_select_plan(ctypes.byref(c), ctypes.byref(q), 655, *args) == tsd.TSD_OK
    assert (f.value, n.value) == (1, 4)
    assert lib.tsd_topk_select_plan(ctypes.byref(c), ctypes.byref(q), 0, *args) == tsd.TSD_ERR_INVALID_ARGUMENT
    assert lib.tsd_topk_select_plan(ctypes.byref(c), ctypes.byref(q), 655, None,
                                    ctypes.byref(n)) == tsd.TSD_ERR_INVALID_ARGUMENT
    bad = make_cache(head_dim=64)
    assert lib.tsd_topk_select_plan(ctypes.byref(bad), ctypes.byref(q), 655, *args) == tsd.TSD_ERR_UNSUPPORTED


def test_topk_filter_not_taken_past_the_candidate_bitmap(lib, monkeypatch):
    """Lists longer than the candidate selection's 128K-token bitmaps would all fall back to the
    recomputed rows, so a call with a longer max_seq_len takes the form over score rows, even
    with the filter forced."""
    monkeypatch.setenv("TSD_TOPK_FILTER", "1")
    f, n = ctypes.c_int32(), ctypes.c_int32()
    c = make_cache(batch=8, max_pages=16384, num_pages=8 * 16384, max_seq_len=262144)
    q = make_queries()
    assert lib.tsd_topk_select_plan(ctypes.byref(c), ctypes.byref(q), 655, ctypes.byref(f), ctypes.byref(n)) == tsd.TSD_OK
    assert (f.value, n.value) == (0, 2)


def test_topk_workspace_holds_the_filter_regions_only_when_the_filter_can_run(lib, monkeypatch):
    """The exact indexer's workspace grows by the candidate filter's regions -- a threshold key,
    8192 (key, index) candidate slots, a (kv_len, k) pair and a queue entry per list -- only
    for shapes and k where the filter can run: the ragged shape at k = 2622 (filtered) against
    k = 20000 (too many candidates for the buffer); the scores and samples are the same size."""
    monkeypatch.delenv("TSD_TOPK_FILTER", raising=False)
    monkeypatch.delenv("TSD_SCORE_KERNEL", raising=False)
    rc = make_cache(batch=32, max_pages=8192, num_pages=32 * 8192, max_seq_len=131072)
    rq = make_queries(tokens=128, q_indptr=FAKE + 0x800000, max_tokens=4)
    with_filter = lib.tsd_topk_workspace_size(ctypes.byref(rc), ctypes.byref(rq), 2622)
    without = lib.tsd_topk_workspace_size(ctypes.byref(rc), ctypes.byref(rq), 20000)
    lists = 128 * 32
    a256 = lambda n: (n + 255) // 256 * 256
    assert with_filter - without == a256(lists * 4) + a256(lists * 8192 * 8) + a256(lists * 8) + a256(lists * 4)
    c, q = make_cache(), make_queries()   # 256 lists of 32K tokens: rows stay in L2, no filter
    monkeypatch.setenv("TSD_TOPK_FILTER", "1")
    forced = lib.tsd_topk_workspace_size(ctypes.byref(c), ctypes.byref(q), 655)
    monkeypatch.delenv("TSD_TOPK_FILTER")
    assert forced - lib.tsd_topk_workspace_size(ctypes.byref(c), ctypes.byref(q), 655) == \
        a256(256 * 4) + a256(256 * 8192 * 8) + a256(256 * 8) + a256(256 * 4)
