/*
 * tsd.h -- C ABI of the B200 context-sparse decode attention library (libtsd.so).
 *
 * The operations come from "Inference Time Context Sparsity: Illusion or
 * Opportunity?" (gist.science technical summary, section 2 "Oracle Top-K" and
 * "Hardware implementation", section 3.C "Kernel speed-ups" and "Bandwidth
 * efficiency"):
 *   - tsd_topk_select : exact top-k token selection per (query token, q head)
 *                       over the whole KV cache ("Oracle Top-K");
 *   - tsd_sparse_decode: decode attention that reads only the selected K/V rows,
 *                       which may differ per token, per query and per head
 *                       (traffic O(k d) instead of O(N d));
 *   - tsd_dense_decode : the dense decode attention it is measured against
 *                       (O(N d) traffic).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are DEVICE pointers unless the comment says "host".  The caller
 *    owns every buffer; the library allocates nothing and keeps no state
 *    between calls.  Calls are asynchronous on the given stream.
 *  - head_dim must be 128.  num_q_heads must be a multiple of num_kv_heads;
 *    q head h reads kv head h / (num_q_heads / num_kv_heads).
 *  - Host-checkable errors return a status without launching anything.
 *    Problems only the device can see (an index outside [0, kv_len), a list
 *    that is not ascending, a page id outside [0, num_pages), a sequence length
 *    above max_seq_len) never fault: the offending entry is skipped and a bit is
 *    OR-ed into the status word at the start of the workspace; read it with
 *    tsd_read_device_status.
 *  - Workspace: each call takes (ws, ws_bytes) of at least the size returned by
 *    the matching *_workspace_size function.  Its first part must be zero when a
 *    call starts; every call leaves it zero again, so zero it once (cudaMemset or
 *    tsd_workspace_init) after allocating it and again whenever the cache or
 *    query shape changes.  Calls that share a workspace must not overlap in time.
 *  - Thread safety: calls with distinct workspaces may run concurrently.
 */
#ifndef TSD_H_
#define TSD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tsd_stream_t; /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
  TSD_OK = 0,
  TSD_ERR_INVALID_ARGUMENT = 1,    /* null pointer, negative size, inconsistent shape */
  TSD_ERR_UNSUPPORTED = 2,         /* head_dim != 128, page_size not a power of two, dtype */
  TSD_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_size result */
  TSD_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  TSD_ERR_DEVICE_STATUS = 5        /* returned by tsd_read_device_status when a bit is set */
} tsd_status;

typedef enum { TSD_BF16 = 0, TSD_F32 = 1 } tsd_dtype;

/* Bits of the device status word. */
enum {
  TSD_DEV_BAD_INDEX = 1u << 0, /* an index entry was < -1 or >= kv_len of its query; skipped */
  TSD_DEV_UNSORTED = 1u << 1,  /* an index list was not ascending where it was read          */
  TSD_DEV_BAD_PAGE = 1u << 2,  /* a page-table entry was outside [0, num_pages); row skipped */
  TSD_DEV_BAD_SEQ = 1u << 3,   /* seq_len outside [0, max_seq_len] or a bad q_indptr; the
                                  outputs of the affected sequence are not written          */
  TSD_DEV_TIMEOUT = 1u << 4    /* a bounded wait inside a kernel gave up (an asynchronous
                                  copy never completed); the results are not valid          */
};

typedef enum {
  /* k, v: [num_pages][num_kv_heads][page_size][head_dim] bf16 ("HND" pages).
     Token i of sequence b lives in page page_table[b * max_pages_per_seq + i / page_size],
     slot i % page_size.  page_size must be a power of two. */
  TSD_LAYOUT_PAGED = 0,
  /* k, v: [batch][num_kv_heads][max_seq_len][head_dim] bf16; page_table must be NULL. */
  TSD_LAYOUT_CONTIGUOUS = 1
} tsd_layout;

/* A bf16 KV cache. */
typedef struct {
  const void* k;               /* device, bf16, layout above */
  const void* v;               /* device, bf16, same layout as k */
  int32_t layout;              /* tsd_layout */
  int32_t num_kv_heads;        /* Hkv >= 1 */
  int32_t head_dim;            /* must be 128 */
  int32_t page_size;           /* paged: power of two >= 1; contiguous: ignored */
  const int32_t* page_table;   /* device int32 [batch][max_pages_per_seq] (paged), else NULL */
  int32_t max_pages_per_seq;   /* paged: >= ceil(max_seq_len / page_size) */
  int64_t num_pages;           /* paged: number of physical pages in k and v */
  const int32_t* seq_lens;     /* device int32 [batch]: tokens cached per sequence */
  int32_t batch;               /* number of sequences B >= 1 */
  int32_t max_seq_len;         /* host bound on every seq_lens[b] (>= 1) */
} tsd_kv_cache;

/* The decode queries of one step. */
typedef struct {
  const void* q;               /* device [num_tokens][num_q_heads][head_dim], q_dtype */
  int32_t q_dtype;             /* TSD_BF16 or TSD_F32 */
  int32_t num_q_heads;         /* Hq, a multiple of num_kv_heads */
  int32_t num_tokens;          /* T: query tokens over all sequences */
  const int32_t* q_indptr;     /* device int32 [batch+1]: tokens of sequence b are
                                  q_indptr[b] .. q_indptr[b+1]-1; NULL means one token per
                                  sequence (T == batch) */
  int32_t max_tokens_per_seq;  /* host bound on q_indptr[b+1]-q_indptr[b] (1 when q_indptr is NULL) */
  int32_t causal;              /* nonzero: token j of the n_b tokens of sequence b sees
                                  kv_len = seq_lens[b] - n_b + j + 1 tokens; zero: it sees
                                  all seq_lens[b] tokens */
  float sm_scale;              /* softmax scale, usually 1/sqrt(head_dim) */
} tsd_queries;

/* Library version as major*10000 + minor*100 + patch. */
int32_t tsd_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* tsd_status_string(tsd_status s);

/* Zero `bytes` bytes of a workspace on `stream` (cudaMemsetAsync). */
tsd_status tsd_workspace_init(void* ws, size_t bytes, tsd_stream_t stream);

/* Host: bytes of workspace tsd_topk_select needs for these shapes (0 on invalid input). */
size_t tsd_topk_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max);

/*
 * Exact top-k token selection ("Oracle Top-K", pages section 2).
 * For each query token t (of sequence b) and q head h (kv head g):
 *   s_i = sum_d q[t,h,d] * K[b,g,i,d], accumulated in fp32 from bf16 inputs, for i < kv_len(t);
 *   keep the k_t = min(k, kv_len(t)) tokens with the largest s_i, ties to the lower index,
 *   where k = k_per_token[t] if k_per_token is non-NULL, else k_max (k_per_token[t] is
 *   clamped to [0, k_max]).  The softmax scale is not applied (it does not change the order).
 * out_idx  : device int32 [T][Hq][k_max]; the k_t kept token indices in ascending order,
 *            then -1 up to k_max.
 * out_count: device int32 [T][Hq] or NULL; receives k_t.
 * k_max >= 1.  Errors: INVALID_ARGUMENT, UNSUPPORTED, WORKSPACE_TOO_SMALL, CUDA.
 * Two forms give the same lists (tsd_topk_select_plan says which a call takes): the scores of
 * every visible token written to the workspace and selected from there, or -- bf16 queries,
 * score rows too large to stay in L2, k small enough -- a candidate filter: a strided sample of
 * every list sets a threshold below which no top-k score can lie (with overwhelming
 * probability; a list whose sample misled it is recomputed in full, so the result is exact
 * either way), the scoring keeps only the scores that reach it, and the selection works on
 * those.  The workspace (tsd_topk_workspace_size) holds both forms' buffers.
 */
tsd_status tsd_topk_select(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                           const int32_t* k_per_token, int32_t* out_idx, int32_t* out_count,
                           void* ws, size_t ws_bytes, tsd_stream_t stream);

/* Host: bytes of workspace tsd_sparse_decode needs for these shapes on the current device
 * (0 on invalid input).  The work split, and so the size, depends on the device's SM count:
 * size the workspace with the device that will run the calls current (148 SMs are assumed
 * when no device can be queried). */
size_t tsd_sparse_decode_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries,
                                        int32_t k_max);

/* Host: the work decomposition tsd_sparse_decode would use for these shapes on the current
 * device, for diagnostics and benchmarks: *persistent = 1 for the persistent kernel
 * (sparse_stream_kernel: every warp takes (list, chunk) tasks from a counter until none is
 * left), 0 for the one-task-per-warp kernel (sparse_decode_kernel: one wave of CTAs);
 * *entries_per_task = index entries per task; *tasks_per_list = tasks (split-K partials) per
 * list.  Device pointers may be NULL.  Errors: INVALID_ARGUMENT, UNSUPPORTED (as
 * tsd_sparse_decode's host checks). */
tsd_status tsd_sparse_decode_plan(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                  int32_t* persistent, int32_t* entries_per_task, int32_t* tasks_per_list);

/* The form tsd_topk_select takes for these shapes and k_max (the exact indexer of the pages'
 * section 2, "Oracle Top-K").  *filtered = 1 for the candidate-filtered form: a sample pre-pass
 * sets a per-list threshold, the scoring kernel keeps only the scores that reach it, and the
 * selection works on those (exact in either form; chosen for bf16 queries when the score rows
 * would not stay in L2 and the expected candidates fit).  0 for the form over full score rows.
 * *kernels = the kernels one call launches (4 or 2).  The environment variable TSD_TOPK_FILTER
 * (0, 1 or rescore) overrides the choice, as it does for tsd_topk_select.  Device pointers may
 * be NULL.  Errors: INVALID_ARGUMENT, UNSUPPORTED (as tsd_topk_select's host checks). */
tsd_status tsd_topk_select_plan(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                int32_t* filtered, int32_t* kernels);

/*
 * Sparse decode attention over per-(token, head) index lists (pages section 2,
 * "Hardware implementation"; section 3.C).  For each query token t and q head h:
 *   z_i = sm_scale * q[t,h] . K[b,g,i]   for every entry i of idx[t][h][0..k_max)
 *   out[t,h] = sum_i exp(z_i - M) V[b,g,i] / sum_i exp(z_i - M),   M = max_i z_i
 *   lse[t,h] = M + ln sum_i exp(z_i - M)       (natural log of the scaled scores)
 * idx: device int32 [T][Hq][k_max].  Each list holds token indices in non-decreasing order
 *   (as tsd_topk_select writes them), followed by -1 padding; every entry is one term, so a
 *   repeated token counts once per occurrence.  A list ends at its first -1: the entries after
 *   it are padding and may be left unread.  Entries >= kv_len(t) or < -1 are skipped and set
 *   TSD_DEV_BAD_INDEX; an observed descending pair sets TSD_DEV_UNSORTED (the result for such a
 *   list is unspecified).  Rows shared by several lists of one kv head (the q heads of a GQA
 *   group and the query tokens of one sequence) are loaded from memory once.
 * out: device [T][Hq][128] of out_dtype (TSD_BF16 or TSD_F32).  An empty list gives zeros.
 * lse: device f32 [T][Hq] or NULL; -inf for an empty list.
 */
tsd_status tsd_sparse_decode(const tsd_kv_cache* cache, const tsd_queries* queries,
                             const int32_t* idx, int32_t k_max, void* out, int32_t out_dtype,
                             float* lse, void* ws, size_t ws_bytes, tsd_stream_t stream);

/* Host: bytes of workspace tsd_sparse_decode_host needs: the tsd_sparse_decode workspace
 * followed by device staging for q, the index lists, out and lse (0 on invalid input). */
size_t tsd_sparse_decode_host_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries,
                                             int32_t k_max, int32_t out_dtype);

/*
 * tsd_sparse_decode for per-step inputs and outputs that live in host memory, in one call:
 * queries->q, idx, out and lse may be host pointers (page-locked memory lets the copies run
 * asynchronously; pageable memory works but each copy then waits for the host).  On `stream`
 * the call enqueues the copies of q and idx into device staging inside `ws`, the sparse decode,
 * and the copies of out (and lse, when non-NULL) back, and returns before they finish:
 * synchronise the stream before reading out or lse, or before reusing q or idx.  The copy
 * direction follows from the pointers (unified addressing), so device pointers work too.  The
 * cache (k, v, page_table, seq_lens) and queries->q_indptr stay device pointers.
 * ws: at least tsd_sparse_decode_host_workspace_size bytes; its leading region follows the
 * tsd_sparse_decode rules.  Errors: as tsd_sparse_decode (nothing is enqueued on a
 * host-checkable error); CUDA if a copy cannot be enqueued.
 */
tsd_status tsd_sparse_decode_host(const tsd_kv_cache* cache, const tsd_queries* queries,
                                  const int32_t* idx, int32_t k_max, void* out, int32_t out_dtype,
                                  float* lse, void* ws, size_t ws_bytes, tsd_stream_t stream);

/*
 * Weighted sparse decode: as tsd_sparse_decode, with entry i of list (t, h) weighted by
 * w = exp(logw[t][h][i]): out = sum_i w_i e^{z_i} V_i / sum_i w_i e^{z_i} and
 * lse = ln sum_i w_i e^{z_i}, z_i = sm_scale q.K_i.  logw: device fp32 [T][Hq][k_max], read
 * only where idx >= 0.  Used with tsd_stochastic_select (the estimator of vAttention-style
 * sampling); same workspace as tsd_sparse_decode.  Errors: as tsd_sparse_decode, plus
 * INVALID_ARGUMENT for a NULL logw.
 */
tsd_status tsd_sparse_decode_weighted(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                      const float* logw, int32_t k_max, void* out, int32_t out_dtype, float* lse,
                                      void* ws, size_t ws_bytes, tsd_stream_t stream);

/*
 * vAttention-style stochastic selection ("Inference Time Context Sparsity: Illusion or
 * Opportunity?", gist.science summary, section 2: stochastic index selection with vAttention,
 * against deterministic top-k).  The pages give no sampling scheme; per (t, h) this keeps the
 * top-k list S given in topk_idx (ascending, -1 padded, as tsd_topk_select writes it) and adds
 * m' = min(m, |R|) tokens of R = [0, kv_len) minus S drawn uniformly without replacement by
 * Floyd's algorithm: step j = |R| - m' .. |R| - 1 keeps rank u[t][h][j - |R| + m'] mod (j + 1),
 * or j when that rank is already kept; rank r of R is its r-th smallest token.
 * u: device uint32 [T][Hq][m], random words supplied by the caller.  Output (device, width
 * k_max + m per list): out_idx int32 -- S and the sample merged ascending, then -1; out_logw
 * fp32 -- 0 for S, ln(|R| / m') for sampled entries (the Horvitz-Thompson weight).  A topk_idx
 * list that is not ascending or reaches kv_len is flagged in *status (TSD_DEV_BAD_INDEX, if
 * status is not NULL) and treated as empty.  Errors: INVALID_ARGUMENT, UNSUPPORTED (m > 1024), CUDA.
 */
tsd_status tsd_stochastic_select(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* topk_idx,
                                 int32_t k_max, const uint32_t* u, int32_t m, int32_t* out_idx, float* out_logw,
                                 uint32_t* status, tsd_stream_t stream);

/* Host: bytes of workspace tsd_dense_decode needs for these shapes on the current device
 * (0 on invalid input).  As for sparse decode, the split into windows depends on the device's
 * SM count (148 assumed when no device can be queried). */
size_t tsd_dense_decode_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries);

/*
 * Dense decode attention (the baseline of pages section 3.C): tsd_sparse_decode with the
 * list {0, 1, ..., kv_len(t)-1} for every (t, h), streamed page by page.
 * out, lse: as tsd_sparse_decode.
 */
tsd_status tsd_dense_decode(const tsd_kv_cache* cache, const tsd_queries* queries, void* out,
                            int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                            tsd_stream_t stream);

/* Host: bytes of workspace tsd_decode_step needs for these shapes on the current device: the
 * larger of the top-k and sparse-decode workspaces (they share one region, used one after the
 * other), plus room for the index lists when the caller passes no out_idx (0 on invalid input). */
size_t tsd_decode_step_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max);

/*
 * One decode step of the method: the exact top-k indexer followed by sparse decode over the
 * rows it selected ("Inference Time Context Sparsity: Illusion or Opportunity?", section 3.C,
 * "Indexing overhead": the indexer's cost is part of the end-to-end step).  It computes
 *   idx = tsd_topk_select(cache, queries, k_max, k_per_token)
 *   out, lse = tsd_sparse_decode(cache, queries, idx)
 * with both calls on one workspace and on `stream`: the fp32 score rows of the first are read
 * by its own selection kernel (the K stream is loaded evict-first, so they stay in L2), and
 * the second reuses the same bytes for its split-K partials.  Nothing is allocated and the
 * host never waits, so the step can be captured into one CUDA graph and replayed.
 * out_idx  : device int32 [T][Hq][k_max] receiving the selected lists, or NULL to keep them
 *            inside `ws`.
 * out_count: device int32 [T][Hq] or NULL; receives min(k_t, kv_len(t)).
 * out, out_dtype, lse: as tsd_sparse_decode.
 * ws: at least tsd_decode_step_workspace_size bytes, 256-byte aligned, zeroed once
 *   (tsd_workspace_init); every call leaves its leading region zero again.
 * Errors: as tsd_topk_select and tsd_sparse_decode (nothing is launched on a host-checkable
 * error); device-detected problems set bits in the status word at the start of `ws`.
 */
tsd_status tsd_decode_step(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                           const int32_t* k_per_token, int32_t* out_idx, int32_t* out_count, void* out,
                           int32_t out_dtype, float* lse, void* ws, size_t ws_bytes, tsd_stream_t stream);

/*
 * Sparse decode for callers that cannot allocate device memory.  The pages have no
 * counterpart to this entry point: it exists for callers such as a plugin running inside
 * another runtime that owns all device memory, or a decode loop that must not call
 * cudaMalloc (which synchronizes the device) and cannot pass a workspace down to here.
 * It computes exactly what tsd_sparse_decode computes (same arguments and results) but
 * allocates nothing and takes no workspace: its scratch lives in a 16 MiB array inside the
 * library, which every GPU that loads the library holds until the process exits.
 *  - Shapes whose scratch exceeds 16 MiB return TSD_ERR_WORKSPACE_TOO_SMALL without
 *    launching (16 MiB covers e.g. 8 sequences x 32 q heads at k = 655).
 *  - The first call on each device looks up the array's device address with that device
 *    current and keeps it for later calls; make that first call before any stream capture.
 *    A cudaDeviceReset destroys the array with the context: the kept address is then stale,
 *    so do not call this entry point on a device after resetting it in the same process.
 *  - Every call shares the one array and clears its status word and merge counters on
 *    `stream` before launching: calls that overlap on the GPU (other streams, other host
 *    threads) race and must be serialized by the caller.
 *  - status: device uint32 the kernel ORs TSD_DEV_* bits into, or NULL to drop them (the
 *    caller clears it; it cannot be read with tsd_read_device_status).
 */
tsd_status tsd_sparse_decode_static_ws(const tsd_kv_cache* cache, const tsd_queries* queries,
                                       const int32_t* idx, int32_t k_max, void* out, int32_t out_dtype,
                                       float* lse, uint32_t* status, tsd_stream_t stream);

/*
 * Copy the device status word of `ws` to *flags (host), clear it, and synchronize `stream`.
 * Returns TSD_OK when no bit was set, TSD_ERR_DEVICE_STATUS when one was, TSD_ERR_CUDA on a
 * CUDA failure.
 */
tsd_status tsd_read_device_status(void* ws, tsd_stream_t stream, uint32_t* flags);

/*
 * tsd_topk_select, also returning the kept tokens' scores: out_scores device fp32
 * [T][Hq][k_max], the unscaled q.K of each kept index (-inf in the padding; -0 as +0).
 * Errors: as tsd_topk_select, plus INVALID_ARGUMENT for a NULL out_scores.
 */
tsd_status tsd_topk_select_scores(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                  const int32_t* k_per_token, int32_t* out_idx, float* out_scores,
                                  int32_t* out_count, void* ws, size_t ws_bytes, tsd_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Context-parallel decode over a token-sharded cache.  Not on the pages: a way to run the
 * path over contexts split across GPUs.  Rank r holds a token range of every sequence, the
 * ranges in rank order.  Each rank:
 *   1. runs tsd_topk_select_scores on its shard (single-token decode, or non-causal);
 *   2. after the caller gathers every rank's (local index, score) candidates rank-major,
 *      keeps the global top-k among them with tsd_cp_merge_select;
 *   3. decodes its shard over the entries it keeps, with fp32 output and lse;
 *   4. after the caller gathers the P (output, lse) pairs, merges them with
 *      tsd_merge_partials.
 * The global top-k lies in the union of the local top-k lists, so the result equals the
 * single-GPU path's.
 * --------------------------------------------------------------------------------------- */

/*
 * cand_idx, cand_scores: device [ranks][lists][k_cand]: each rank's shard-local token indices
 * (ascending, -1 padding) and their scores, rank r's token range preceding rank r + 1's.
 * Per list, keeps the k largest scores among all candidates (k = k_per_list[list] if not
 * NULL, else k; ties to the lower global index) and writes the kept candidates of rank
 * my_rank -- its local indices -- ascending, -1 padded, to out_idx [lists][k_out]; if more than
 * k_out are kept there the rest are dropped and TSD_DEV_BAD_INDEX is set in *status (if not
 * NULL).  ranks x k_cand <= 16384.  Errors: INVALID_ARGUMENT, UNSUPPORTED, CUDA.
 */
tsd_status tsd_cp_merge_select(const int32_t* cand_idx, const float* cand_scores, int32_t ranks, int64_t lists,
                               int32_t k_cand, const int32_t* k_per_list, int32_t k, int32_t my_rank,
                               int32_t* out_idx, int32_t k_out, uint32_t* status, tsd_stream_t stream);

/*
 * Merge P partial decode results of the same rows: out_parts device fp32 [parts][rows][128]
 * (each normalised over its own entries), lse_parts [parts][rows].  out = sum_p w_p out_p /
 * sum_p w_p with w_p = exp(lse_p - max_p lse_p); lse = max + ln sum_p w_p; rows whose parts
 * are all -inf get out = 0 and lse = -inf.  out: device [rows][128] of out_dtype; lse: device
 * fp32 [rows] or NULL.  16-byte aligned.  Errors: INVALID_ARGUMENT, UNSUPPORTED, CUDA.
 */
tsd_status tsd_merge_partials(int32_t parts, int64_t rows, const float* out_parts, const float* lse_parts, void* out,
                              int32_t out_dtype, float* lse, tsd_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Label-channel approximate indexer (Double-Sparsity-style).
 *
 * The pages ("Inference Time Context Sparsity: Illusion or Opportunity?", gist.science
 * summary, section 3.C "Indexing overhead") price the indexer in front of sparse decode by
 * simulating Double Sparsity: every token is scored with only a few "label" channels of
 * its key, held in a compact cache, and the top k of those approximate scores are kept.
 * The pages fix neither the channel count nor the choice; this library takes r channels
 * per kv head (r in {8, 16, 32}) with the largest total |q_d K_{i,d}| over a calibration
 * set (ties to the lower channel index), in ascending order.
 * --------------------------------------------------------------------------------------- */

/* Host: bytes of the label cache for `cache` and r channels: one row of r bf16 values per K
 * row, same layout and row numbering as K (paged: [num_pages][Hkv][page_size][r];
 * contiguous: [B][Hkv][max_seq_len][r]).  0 on invalid input. */
size_t tsd_label_cache_bytes(const tsd_kv_cache* cache, int32_t r);

/* Host: workspace bytes of tsd_label_channels (0 on invalid input). */
size_t tsd_label_channels_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries);

/*
 * Offline calibration: choose r label channels per kv head from the queries and the cache.
 * importance[g][d] = sum over sequences b of (sum over the queries t of b and q heads h of
 * group g of |q[t,h,d]|) x (sum over tokens i < seq_lens[b] of |K[b,g,i,d]|), accumulated in
 * fp64 in a fixed order (deterministic); the r largest per g, ties to the lower d.
 * channels: device int32 [Hkv][r], ascending per kv head.  The first 4 bytes of ws receive
 * the device status (bad page or length); the workspace needs no zeroing.
 * Errors: INVALID_ARGUMENT (r not in {8, 16, 32}, null pointers), WORKSPACE_TOO_SMALL, CUDA.
 */
tsd_status tsd_label_channels(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t r,
                              int32_t* channels, void* ws, size_t ws_bytes, tsd_stream_t stream);

/*
 * Build the label cache: label_k[row][j] = K[row][channels[g][j]] for every K row (rows of
 * unused slots included).  channels: device int32 [Hkv][r] in [0, 128) (an entry outside
 * that range reads channel 0 and sets TSD_DEV_BAD_INDEX in *status).  label_k: device, at
 * least tsd_label_cache_bytes(cache, r) bytes, 16-byte aligned.  status: device uint32 or
 * NULL.  Errors: INVALID_ARGUMENT, UNSUPPORTED (r), CUDA.
 */
tsd_status tsd_label_cache_build(const tsd_kv_cache* cache, const int32_t* channels, int32_t r, void* label_k,
                                 uint32_t* status, tsd_stream_t stream);

/*
 * Approximate top-k: as tsd_topk_select, but the score of token i for (t, h) is
 * s~_i = sum over j < r of q[t,h,channels[g][j]] * label_k[row(i)][j] (unscaled fp32), and
 * the k largest s~ are kept (ties to the lower index, ascending, -1 padded).  The cache
 * supplies the page table, lengths and shapes; label_k is the tsd_label_cache_build output
 * for the same channels.  Workspace: tsd_topk_workspace_size bytes, zeroed as described
 * above.  Errors: as tsd_topk_select, plus UNSUPPORTED for r not in {8, 16, 32}.
 */
tsd_status tsd_topk_select_label(const tsd_kv_cache* cache, const void* label_k, const int32_t* channels,
                                 int32_t r, const tsd_queries* queries, int32_t k_max, const int32_t* k_per_token,
                                 int32_t* out_idx, int32_t* out_count, void* ws, size_t ws_bytes,
                                 tsd_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TSD_H_ */
