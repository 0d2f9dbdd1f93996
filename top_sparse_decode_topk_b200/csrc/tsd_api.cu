// extern "C" entry points of libtsd: host-side validation, work decomposition,
// workspace layout and kernel launches.  See include/tsd.h for the contract.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "tsd.h"
#include "tsd_common.cuh"
#include "tsd_plan.h"
#include "tsd_filter.cuh"

#include "tsd_args.h"
#include "tsd_kvtile.cuh"

namespace tsd {
cudaError_t launch_sparse_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream, bool dependent);
cudaError_t launch_dense_decode(const DecodeArgs& a, const KvMaps& maps, int batch, int hkv, cudaStream_t stream);
cudaError_t launch_topk(const TopkArgs& a, const KvMaps& maps, int nwin, int batch, int hkv, int num_lists,
                        cudaStream_t stream);
size_t label_channels_ws_bytes(int64_t batch, int64_t hkv);
cudaError_t launch_label_channels(const KvView& kv, const QView& qv, int r, int32_t* channels, void* ws,
                                  cudaStream_t stream);
cudaError_t launch_label_build(const KvView& kv, const int32_t* channels, int r, int64_t rows, uint16_t* label,
                               uint32_t* status, cudaStream_t stream);
cudaError_t launch_stochastic_select(const KvView& kv, const QView& qv, const int32_t* top, int k_max,
                                     const uint32_t* u, int m, int32_t* out_idx, float* out_logw, uint32_t* status,
                                     cudaStream_t stream);
cudaError_t launch_cp_merge_select(const int32_t* cand_idx, const float* cand_score, int P, int64_t lists, int kc,
                                   const int32_t* k_per_list, int k, int my_rank, int32_t* out, int k_out,
                                   uint32_t* status, cudaStream_t stream);
int cp_max_candidates();
cudaError_t launch_merge_partials(int P, int64_t rows, const float* out_parts, const float* lse_parts, void* out,
                                  int out_f32, float* lse, cudaStream_t stream);
cudaError_t launch_label_topk(const TopkArgs& a, const uint16_t* label, const int32_t* channels, int r, int nwin,
                              int batch, int hkv, int num_lists, cudaStream_t stream);
}  // namespace tsd

using namespace tsd;

namespace {

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int log2i(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

// Host validation of the descriptors; fills the kernel views and shape summary.
tsd_status check_inputs(const tsd_kv_cache* c, const tsd_queries* q, KvView* kv, QView* qv, Shapes* sh) {
  if (c == nullptr || q == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  if (c->head_dim != kHeadDim) return TSD_ERR_UNSUPPORTED;
  if (c->k == nullptr || c->v == nullptr || c->seq_lens == nullptr || q->q == nullptr)
    return TSD_ERR_INVALID_ARGUMENT;
  if (c->batch < 1 || c->num_kv_heads < 1 || c->max_seq_len < 1) return TSD_ERR_INVALID_ARGUMENT;
  if (q->num_q_heads < 1 || q->num_q_heads % c->num_kv_heads != 0) return TSD_ERR_INVALID_ARGUMENT;
  if (q->num_tokens < 1) return TSD_ERR_INVALID_ARGUMENT;
  if (q->q_dtype != TSD_BF16 && q->q_dtype != TSD_F32) return TSD_ERR_UNSUPPORTED;
  int max_tokens = q->max_tokens_per_seq;
  if (q->q_indptr == nullptr) {
    if (q->num_tokens != c->batch) return TSD_ERR_INVALID_ARGUMENT;
    max_tokens = 1;
  } else if (max_tokens < 1 || max_tokens > q->num_tokens) {
    return TSD_ERR_INVALID_ARGUMENT;
  }
  if (!(q->sm_scale > 0.f) || q->sm_scale != q->sm_scale) return TSD_ERR_INVALID_ARGUMENT;
  // 16-byte alignment of the row streams
  if (((uintptr_t)c->k & 15) || ((uintptr_t)c->v & 15) || ((uintptr_t)q->q & 15)) return TSD_ERR_INVALID_ARGUMENT;

  memset(kv, 0, sizeof(*kv));
  kv->k = static_cast<const uint16_t*>(c->k);
  kv->v = static_cast<const uint16_t*>(c->v);
  kv->seq_lens = c->seq_lens;
  kv->hkv = c->num_kv_heads;
  kv->max_seq_len = c->max_seq_len;
  kv->batch = c->batch;
  if (c->layout == TSD_LAYOUT_PAGED) {
    if (c->page_table == nullptr || !is_pow2(c->page_size)) return c->page_table ? TSD_ERR_UNSUPPORTED : TSD_ERR_INVALID_ARGUMENT;
    if ((int64_t)c->max_pages_per_seq * c->page_size < c->max_seq_len) return TSD_ERR_INVALID_ARGUMENT;
    if (c->num_pages < 1) return TSD_ERR_INVALID_ARGUMENT;
    // physical rows are addressed with 32-bit row numbers
    if ((double)c->num_pages * c->num_kv_heads * c->page_size >= 4294967295.0) return TSD_ERR_UNSUPPORTED;
    kv->page_table = c->page_table;
    kv->page_shift = log2i(c->page_size);
    kv->max_pages = c->max_pages_per_seq;
    kv->num_pages = c->num_pages;
  } else if (c->layout == TSD_LAYOUT_CONTIGUOUS) {
    if (c->page_table != nullptr) return TSD_ERR_INVALID_ARGUMENT;
    if ((double)c->batch * c->num_kv_heads * c->max_seq_len >= 4294967295.0) return TSD_ERR_UNSUPPORTED;
    kv->page_table = nullptr;
    kv->num_pages = c->batch;
  } else {
    return TSD_ERR_INVALID_ARGUMENT;
  }
  memset(qv, 0, sizeof(*qv));
  qv->q = q->q;
  qv->q_f32 = q->q_dtype == TSD_F32;
  qv->hq = q->num_q_heads;
  qv->num_tokens = q->num_tokens;
  qv->q_indptr = q->q_indptr;
  qv->max_tokens = max_tokens;
  qv->causal = q->causal != 0;
  qv->sm_scale = q->sm_scale;

  sh->batch = c->batch;
  sh->hkv = c->num_kv_heads;
  sh->hq = q->num_q_heads;
  sh->group = q->num_q_heads / c->num_kv_heads;
  sh->tokens = q->num_tokens;
  sh->max_tokens = max_tokens;
  sh->max_seq_len = c->max_seq_len;
  return TSD_OK;
}

tsd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TSD_OK : TSD_ERR_CUDA; }

// Tensor maps of the K and V caches seen as [rows][128] bf16 with a {64, box_rows} box and
// 128-byte swizzling, for the TMA loads of the dense-tile kernels.  Caches whose pages
// are smaller than 8 tokens do not use them (their tiles are copied with cp.async).
tsd_status make_kv_maps(const tsd_kv_cache* c, KvMaps* maps) {
  memset(maps, 0, sizeof(*maps));
  int64_t rows;
  int box_rows;
  if (c->layout == TSD_LAYOUT_CONTIGUOUS) {
    rows = (int64_t)c->batch * c->num_kv_heads * c->max_seq_len;
    box_rows = 16;
  } else {
    if (c->page_size < 8) return TSD_OK;
    rows = c->num_pages * c->num_kv_heads * c->page_size;
    box_rows = c->page_size < 16 ? c->page_size : 16;
  }
  if (rows >= (int64_t)1 << 31) return TSD_ERR_UNSUPPORTED;
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (encode == nullptr) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return TSD_ERR_CUDA;
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const void* ptrs[2] = {c->k, c->v};
  CUtensorMap* out[2] = {&maps->k, &maps->v};
  for (int i = 0; i < 2; ++i) {
    const CUresult r = encode(out[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[i]), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return TSD_ERR_CUDA;
  }
  return TSD_OK;
}

}  // namespace

extern "C" {

int32_t tsd_version(void) { return 100; }

const char* tsd_status_string(tsd_status s) {
  switch (s) {
    case TSD_OK: return "TSD_OK";
    case TSD_ERR_INVALID_ARGUMENT: return "TSD_ERR_INVALID_ARGUMENT";
    case TSD_ERR_UNSUPPORTED: return "TSD_ERR_UNSUPPORTED";
    case TSD_ERR_WORKSPACE_TOO_SMALL: return "TSD_ERR_WORKSPACE_TOO_SMALL";
    case TSD_ERR_CUDA: return "TSD_ERR_CUDA";
    case TSD_ERR_DEVICE_STATUS: return "TSD_ERR_DEVICE_STATUS";
  }
  return "TSD_UNKNOWN_STATUS";
}

tsd_status tsd_workspace_init(void* ws, size_t bytes, tsd_stream_t stream) {
  if (ws == nullptr && bytes > 0) return TSD_ERR_INVALID_ARGUMENT;
  if (bytes == 0) return TSD_OK;
  return cuda_status(cudaMemsetAsync(ws, 0, bytes, reinterpret_cast<cudaStream_t>(stream)));
}

static int topk_filter_choice(const Shapes& sh, bool q_f32, bool with_scores, int32_t k_max);
// The top-k workspace layout, with the candidate filter's regions (thresholds, candidates,
// (kv_len, k), queue) only when `filter`: without them those offsets all equal `total`.
static TopkLayout topk_layout_for(const Shapes& sh, bool filter) {
  TopkLayout l = topk_layout(sh);
  if (!filter) l.off_cand = l.off_meta = l.off_queue = l.total = l.off_lo;
  return l;
}
// Whether a top-k workspace for these shapes holds the candidate filter's regions: when the
// filter could run for some call on them (either indexer; the query dtype aside).
static bool topk_filter_space(const Shapes& sh, int32_t k_max) { return topk_filter_choice(sh, false, false, k_max) != 0; }

size_t tsd_topk_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max) {
  KvView kv; QView qv; Shapes sh;
  if (k_max < 1) return 0;
  // shape-only validation: device pointers may be NULL when only sizing
  tsd_kv_cache c = *cache;
  tsd_queries q = *queries;
  static const uint16_t dummy[8] = {0};
  if (c.k == nullptr) c.k = dummy;
  if (c.v == nullptr) c.v = dummy;
  if (c.seq_lens == nullptr) c.seq_lens = reinterpret_cast<const int32_t*>(dummy);
  if (c.layout == TSD_LAYOUT_PAGED && c.page_table == nullptr) c.page_table = reinterpret_cast<const int32_t*>(dummy);
  if (q.q == nullptr) q.q = dummy;
  if (check_inputs(&c, &q, &kv, &qv, &sh) != TSD_OK) return 0;
  return topk_layout_for(sh, topk_filter_space(sh, k_max)).total;
}

// SM count of the current device: the sparse plan sizes its grid to the resident CTAs.  A
// B200's 148 when no device can be queried (host-only sizing calls on a machine without one).
static int current_sm_count() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int cache[kMaxDev] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return 148;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

// Work decomposition of tsd_sparse_decode.  The one-task-per-warp kernel fits its grid to one
// wave of resident CTAs.  The persistent kernel takes the call instead when that plan needs
// more than one wave, or when it fits one wave only by giving every warp a whole list of 256
// entries or more: lists of unequal length then leave the wave waiting on its longest list,
// while the persistent kernel cuts lists into chunks and balances them over all warps.
// TSD_SPARSE_KERNEL=wave|stream forces either form and TSD_SPARSE_CHUNK sets the persistent
// form's entries per task (both for measurements; read at every call, so size the workspace
// under the same setting as the call).
static SparsePlan sparse_plan(const Shapes& sh, int k_max) {
  const int sms = current_sm_count();
  const char* kind = getenv("TSD_SPARSE_KERNEL");
  const char* chunk = getenv("TSD_SPARSE_CHUNK");
  const int e_override = chunk != nullptr ? atoi(chunk) : 0;
  const SparsePlan wave = plan_sparse(sh, k_max, sms);
  bool stream;
  if (kind != nullptr && strcmp(kind, "stream") == 0) {
    stream = true;
  } else if (kind != nullptr && strcmp(kind, "wave") == 0) {
    stream = false;
  } else {
    const int64_t ctas = (sh.batch * sh.hkv * wave.lists * (int64_t)wave.nsplit + kSpTasksPerCta - 1) / kSpTasksPerCta;
    stream = ctas > (int64_t)sms * kSpCtasPerSm || (wave.nsplit == 1 && k_max >= 256);
  }
  return stream ? plan_sparse_stream(sh, k_max, sms, e_override) : wave;
}

static tsd_status sizes_for(const tsd_kv_cache* cache, const tsd_queries* queries, Shapes* sh) {
  if (cache == nullptr || queries == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  KvView kv; QView qv;
  tsd_kv_cache c = *cache;
  tsd_queries q = *queries;
  static const uint16_t dummy[8] = {0};
  if (c.k == nullptr) c.k = dummy;
  if (c.v == nullptr) c.v = dummy;
  if (c.seq_lens == nullptr) c.seq_lens = reinterpret_cast<const int32_t*>(dummy);
  if (c.layout == TSD_LAYOUT_PAGED && c.page_table == nullptr) c.page_table = reinterpret_cast<const int32_t*>(dummy);
  if (q.q == nullptr) q.q = dummy;
  return check_inputs(&c, &q, &kv, &qv, sh);
}

size_t tsd_sparse_decode_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max) {
  Shapes sh;
  if (k_max < 1 || k_max > kMaxSparseK || sizes_for(cache, queries, &sh) != TSD_OK) return 0;
  const SparsePlan p = sparse_plan(sh, k_max);
  return decode_layout(sh, p.nsplit).total;
}

tsd_status tsd_sparse_decode_plan(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                  int32_t* persistent, int32_t* entries_per_task, int32_t* tasks_per_list) {
  Shapes sh;
  if (k_max < 1 || persistent == nullptr || entries_per_task == nullptr || tasks_per_list == nullptr)
    return TSD_ERR_INVALID_ARGUMENT;
  if (k_max > kMaxSparseK) return TSD_ERR_UNSUPPORTED;
  const tsd_status st = sizes_for(cache, queries, &sh);
  if (st != TSD_OK) return st;
  const SparsePlan p = sparse_plan(sh, k_max);
  *persistent = p.stream;
  *entries_per_task = p.entries;
  *tasks_per_list = p.nsplit;
  return TSD_OK;
}

size_t tsd_dense_decode_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries) {
  Shapes sh;
  if (sizes_for(cache, queries, &sh) != TSD_OK) return 0;
  const DensePlan p = plan_dense(sh, (int64_t)current_sm_count() * kDnCtasPerSm);
  return decode_layout(sh, p.nsplit).total;
}

// The exact indexer's candidate filter.  TSD_TOPK_FILTER unset: on when the score rows would not
// stay in L2 (see topk_select_impl); "1": on wherever it can serve the call; "0": off;
// "rescore": on with every threshold disabled, so that every list takes the selection's row
// recomputation (a test hook for that path).
enum { kFilterAuto = -1, kFilterOff = 0, kFilterOn = 1, kFilterRescore = 2 };
static int filter_mode() {
  const char* e = getenv("TSD_TOPK_FILTER");
  if (e == nullptr) return kFilterAuto;
  if (strcmp(e, "0") == 0) return kFilterOff;
  if (strcmp(e, "rescore") == 0) return kFilterRescore;
  return kFilterOn;
}

// Score rows above this many bytes leave L2 between the scoring kernel and the selection, so
// the unfiltered form writes them to DRAM and reads them back; below it they stay in the 126 MB
// L2 and the filter's pre-pass costs more than it saves.
constexpr double kFilterMinRowBytes = 64.0 * 1024 * 1024;

// Whether a list of any length with k <= k_max passes the pre-pass's size test when its
// sample takes every 2^shift-th token: with m = k_max / 2^shift the expected sample count above
// the k-th score is at most m + 1, and r = ceil(m + 1 + 4 sqrt(m + 1) + 4) samples at stride
// 2^shift stand for at most r 2^shift candidates, which must stay within 3/4 of the buffer.
static bool filter_fits(int32_t k_max, int shift) {
  const double m = (double)k_max / (double)(1LL << shift) + 1.0;
  const double r = ceil(m + 4.0 * sqrt(m) + 4.0);
  return r * (double)(1LL << shift) <= (double)kTopkCandCap * 3.0 / 4.0;
}
static bool score_on_tcgen05_host() {
  const char* e = getenv("TSD_SCORE_KERNEL");
  return e != nullptr && strcmp(e, "tcgen05") == 0;
}

// The form of the exact indexer for a call: 0 unfiltered, 1 candidate-filtered, 2 filtered with
// every threshold disabled (TSD_TOPK_FILTER=rescore).
static int topk_filter_choice(const Shapes& sh, bool q_f32, bool with_scores, int32_t k_max) {
  const TopkLayout lay = topk_layout(sh);
  const int fm = filter_mode();
  const double row_bytes = (double)sh.tokens * sh.hq * (double)lay.score_stride * sizeof(float);
  const bool can = !q_f32 && !with_scores && !score_on_tcgen05_host() && sh.max_seq_len <= kTopkCandMaxLen;
  if (fm == kFilterRescore) return can ? 2 : 0;
  if (fm == kFilterOn) return can && filter_fits(k_max, lay.sample_shift + 1) ? 1 : 0;
  if (fm == kFilterAuto)
    return can && filter_fits(k_max, lay.sample_shift + 1) && row_bytes > kFilterMinRowBytes ? 1 : 0;
  return 0;
}

tsd_status tsd_topk_select_plan(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                int32_t* filtered, int32_t* kernels) {
  Shapes sh;
  if (k_max < 1 || filtered == nullptr || kernels == nullptr || queries == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  const tsd_status st = sizes_for(cache, queries, &sh);
  if (st != TSD_OK) return st;
  const int f = topk_filter_choice(sh, queries->q_dtype == TSD_F32, false, k_max);
  *filtered = f != 0 ? 1 : 0;
  *kernels = f != 0 ? 4 : 2;
  return TSD_OK;
}

static tsd_status topk_select_impl(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                   const int32_t* k_per_token, int32_t* out_idx, float* out_scores,
                                   int32_t* out_count, void* ws, size_t ws_bytes, tsd_stream_t stream) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = check_inputs(cache, queries, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  if (k_max < 1 || out_idx == nullptr || ws == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  if (((uintptr_t)ws & 255) != 0) return TSD_ERR_INVALID_ARGUMENT;
  const TopkLayout lay = topk_layout_for(sh, topk_filter_space(sh, k_max));
  if (ws_bytes < lay.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  TopkArgs a;
  memset(&a, 0, sizeof(a));
  a.kv = kv;
  a.qv = qv;
  a.k_max = k_max;
  a.k_per_token = k_per_token;
  a.out_idx = out_idx;
  a.out_count = out_count;
  a.out_scores = out_scores;
  a.scores = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_scores);
  a.score_stride = lay.score_stride;
  a.samples = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_samples);
  a.sample_stride = lay.sample_stride;
  a.sample_shift = lay.sample_shift;
  // The candidate filter (sample pre-pass, per-list threshold, candidate appends while scoring,
  // no score rows) serves bf16 queries with the warp-MMA scoring kernel when k_max is small
  // enough for the candidates to fit; the kept scores' output (tsd_topk_select_scores), fp32
  // queries and larger k take the paths over the full score rows.
  a.filter = topk_filter_choice(sh, qv.q_f32, out_scores != nullptr, k_max);
  if (a.filter) a.sample_shift = lay.sample_shift + 1;   // the pre-pass samples every other sample slot
  a.lo_key = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + lay.off_lo);
  a.cand = reinterpret_cast<uint2*>(static_cast<char*>(ws) + lay.off_cand);
  a.meta = reinterpret_cast<int2*>(static_cast<char*>(ws) + lay.off_meta);
  a.queue = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + lay.off_queue);
  a.queue_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 16);
  a.queue_done = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 20);
  a.cand_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 256);
  // scoring streams K in the dense path's tiles, with its own occupancy
  const DensePlan p = plan_dense(sh, (int64_t)current_sm_count() * kScoreCtasPerSm, kMaxWindowScore);
  a.lists_per_cta = p.lists_per_cta;
  a.list_groups = p.list_groups;
  a.window = p.window;
  a.status = static_cast<uint32_t*>(ws);
  if (a.filter) {
    // the pre-pass: about six CTAs per SM in all, each group's 16-row sample tiles split evenly
    const int64_t groups = sh.batch * sh.hkv * p.list_groups;
    const int64_t tiles = (((int64_t)sh.max_seq_len + (1LL << a.sample_shift) - 1) >> a.sample_shift) / 16 + 1;
    int64_t splits = (6LL * current_sm_count() + groups - 1) / groups;
    a.prepass_splits = (int)(splits < 1 ? 1 : (splits > tiles ? tiles : splits));
    const int64_t qc = 2LL * current_sm_count();   // the selection's CTAs per SM
    a.queue_ctas = (int)(qc < sh.tokens * sh.hq ? qc : sh.tokens * sh.hq);
  }
  KvMaps maps;
  st = make_kv_maps(cache, &maps);
  if (st != TSD_OK) return st;
  return cuda_status(launch_topk(a, maps, p.nsplit, (int)sh.batch, (int)sh.hkv, (int)(sh.tokens * sh.hq),
                                 reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_topk_select(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                           const int32_t* k_per_token, int32_t* out_idx, int32_t* out_count, void* ws,
                           size_t ws_bytes, tsd_stream_t stream) {
  return topk_select_impl(cache, queries, k_max, k_per_token, out_idx, nullptr, out_count, ws, ws_bytes, stream);
}

tsd_status tsd_topk_select_scores(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                  const int32_t* k_per_token, int32_t* out_idx, float* out_scores,
                                  int32_t* out_count, void* ws, size_t ws_bytes, tsd_stream_t stream) {
  if (out_scores == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  return topk_select_impl(cache, queries, k_max, k_per_token, out_idx, out_scores, out_count, ws, ws_bytes, stream);
}

tsd_status tsd_cp_merge_select(const int32_t* cand_idx, const float* cand_scores, int32_t ranks, int64_t lists,
                               int32_t k_cand, const int32_t* k_per_list, int32_t k, int32_t my_rank,
                               int32_t* out_idx, int32_t k_out, uint32_t* status, tsd_stream_t stream) {
  if (cand_idx == nullptr || cand_scores == nullptr || out_idx == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  if (ranks < 1 || lists < 1 || k_cand < 1 || k < 0 || k_out < 1 || my_rank < 0 || my_rank >= ranks)
    return TSD_ERR_INVALID_ARGUMENT;
  if ((int64_t)ranks * k_cand > cp_max_candidates()) return TSD_ERR_UNSUPPORTED;
  return cuda_status(launch_cp_merge_select(cand_idx, cand_scores, ranks, lists, k_cand, k_per_list, k, my_rank,
                                            out_idx, k_out, status, reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_merge_partials(int32_t parts, int64_t rows, const float* out_parts, const float* lse_parts, void* out,
                              int32_t out_dtype, float* lse, tsd_stream_t stream) {
  if (parts < 1 || rows < 1 || out_parts == nullptr || lse_parts == nullptr || out == nullptr)
    return TSD_ERR_INVALID_ARGUMENT;
  if (out_dtype != TSD_BF16 && out_dtype != TSD_F32) return TSD_ERR_UNSUPPORTED;
  if (((uintptr_t)out_parts & 15) != 0 || ((uintptr_t)out & 15) != 0) return TSD_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_merge_partials(parts, rows, out_parts, lse_parts, out, out_dtype == TSD_F32, lse,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

static tsd_status decode_common(const tsd_kv_cache* cache, const tsd_queries* queries, void* out,
                                int32_t out_dtype, float* lse, void* ws, size_t ws_bytes, KvView* kv,
                                QView* qv, Shapes* sh) {
  tsd_status st = check_inputs(cache, queries, kv, qv, sh);
  if (st != TSD_OK) return st;
  if (out == nullptr || ws == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  if (out_dtype != TSD_BF16 && out_dtype != TSD_F32) return TSD_ERR_UNSUPPORTED;
  if (((uintptr_t)ws & 255) != 0) return TSD_ERR_INVALID_ARGUMENT;
  (void)ws_bytes;
  (void)lse;
  return TSD_OK;
}

// `dependent`: launched right after the selection that wrote idx (tsd_decode_step), as its
// programmatic dependent: the decode kernel starts while the selection drains and waits for it
// before its first read.
static tsd_status sparse_decode_impl(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                     const float* logw, int32_t k_max, void* out, int32_t out_dtype, float* lse,
                                     void* ws, size_t ws_bytes, tsd_stream_t stream, bool dependent = false) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = decode_common(cache, queries, out, out_dtype, lse, ws, ws_bytes, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  if (idx == nullptr || k_max < 1) return TSD_ERR_INVALID_ARGUMENT;
  if (k_max > kMaxSparseK) return TSD_ERR_UNSUPPORTED;
  const SparsePlan p = sparse_plan(sh, k_max);
  const DecodeLayout lay = decode_layout(sh, p.nsplit);
  if (ws_bytes < lay.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.kv = kv;
  a.qv = qv;
  a.idx = idx;
  a.logw = logw;
  a.k_max = k_max;
  a.span = p.entries;
  a.nsplit = p.nsplit;
  a.lists_per_cta = p.lists;
  a.list_groups = 1;
  a.out = out;
  a.out_f32 = out_dtype == TSD_F32;
  a.lse = lse;
  a.status = static_cast<uint32_t*>(ws);
  a.counters = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + lay.off_counters);
  a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + lay.off_ml);
  a.part_acc = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_acc);
  a.sched = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 4);
  a.persistent = p.stream;
  return cuda_status(
      launch_sparse_decode(a, (int)sh.batch, (int)sh.hkv, reinterpret_cast<cudaStream_t>(stream), dependent));
}

tsd_status tsd_sparse_decode(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                             int32_t k_max, void* out, int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                             tsd_stream_t stream) {
  return sparse_decode_impl(cache, queries, idx, nullptr, k_max, out, out_dtype, lse, ws, ws_bytes, stream);
}

// tsd_decode_step: the top-k and sparse-decode workspaces overlaid on one region (the score
// rows are dead once the selection has run), then the index lists when the caller keeps none.
struct StepLayout {
  size_t shared, off_idx, total;
};

static bool step_layout(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max, bool own_idx,
                        StepLayout* L) {
  Shapes sh;
  if (k_max < 1 || k_max > kMaxSparseK || sizes_for(cache, queries, &sh) != TSD_OK) return false;
  const size_t topk = topk_layout_for(sh, topk_filter_space(sh, k_max)).total;
  const size_t dec = decode_layout(sh, sparse_plan(sh, k_max).nsplit).total;
  L->shared = align256(topk > dec ? topk : dec);
  L->off_idx = L->shared;
  L->total = L->shared + (own_idx ? align256((size_t)sh.tokens * sh.hq * k_max * sizeof(int32_t)) : 0);
  return true;
}

size_t tsd_decode_step_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max) {
  StepLayout L;
  return step_layout(cache, queries, k_max, true, &L) ? L.total : 0;
}

tsd_status tsd_decode_step(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                           const int32_t* k_per_token, int32_t* out_idx, int32_t* out_count, void* out,
                           int32_t out_dtype, float* lse, void* ws, size_t ws_bytes, tsd_stream_t stream) {
  // every host check of both calls runs before anything is enqueued
  {
    KvView kv; QView qv; Shapes sh;
    tsd_status st = decode_common(cache, queries, out, out_dtype, lse, ws, ws_bytes, &kv, &qv, &sh);
    if (st != TSD_OK) return st;
    if (k_max < 1) return TSD_ERR_INVALID_ARGUMENT;
    if (k_max > kMaxSparseK) return TSD_ERR_UNSUPPORTED;
  }
  StepLayout L;
  if (!step_layout(cache, queries, k_max, out_idx == nullptr, &L)) return TSD_ERR_INVALID_ARGUMENT;
  if (ws_bytes < L.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  int32_t* idx = out_idx != nullptr ? out_idx : reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.off_idx);
  tsd_status st = topk_select_impl(cache, queries, k_max, k_per_token, idx, nullptr, out_count, ws, L.shared, stream);
  if (st != TSD_OK) return st;
  return sparse_decode_impl(cache, queries, idx, nullptr, k_max, out, out_dtype, lse, ws, L.shared, stream, true);
}

// Device staging of tsd_sparse_decode_host, after the sparse-decode workspace.
struct HostStaging {
  size_t off_q, off_idx, off_out, off_lse, total;
};

static bool host_staging(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max, int32_t out_dtype,
                         HostStaging* hs, size_t* decode_bytes) {
  Shapes sh;
  if (k_max < 1 || k_max > kMaxSparseK || sizes_for(cache, queries, &sh) != TSD_OK) return false;
  if (out_dtype != TSD_BF16 && out_dtype != TSD_F32) return false;
  const SparsePlan p = sparse_plan(sh, k_max);
  *decode_bytes = decode_layout(sh, p.nsplit).total;
  const size_t lists = (size_t)queries->num_tokens * queries->num_q_heads;
  size_t off = align256(*decode_bytes);
  hs->off_q = off;
  off += align256(lists * kHeadDim * (queries->q_dtype == TSD_F32 ? 4 : 2));
  hs->off_idx = off;
  off += align256(lists * (size_t)k_max * sizeof(int32_t));
  hs->off_out = off;
  off += align256(lists * kHeadDim * (out_dtype == TSD_F32 ? 4 : 2));
  hs->off_lse = off;
  off += align256(lists * sizeof(float));
  hs->total = off;
  return true;
}

size_t tsd_sparse_decode_host_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t k_max,
                                             int32_t out_dtype) {
  HostStaging hs;
  size_t dec;
  return host_staging(cache, queries, k_max, out_dtype, &hs, &dec) ? hs.total : 0;
}

tsd_status tsd_sparse_decode_host(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                  int32_t k_max, void* out, int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                                  tsd_stream_t stream) {
  if (cache == nullptr || queries == nullptr || queries->q == nullptr || idx == nullptr || out == nullptr ||
      ws == nullptr)
    return TSD_ERR_INVALID_ARGUMENT;
  HostStaging hs;
  size_t dec;
  if (!host_staging(cache, queries, k_max, out_dtype, &hs, &dec)) {
    // report the same status tsd_sparse_decode would
    KvView kv; QView qv; Shapes sh;
    const tsd_status st = check_inputs(cache, queries, &kv, &qv, &sh);
    if (st != TSD_OK) return st;
    if (out_dtype != TSD_BF16 && out_dtype != TSD_F32) return TSD_ERR_UNSUPPORTED;
    return k_max > kMaxSparseK ? TSD_ERR_UNSUPPORTED : TSD_ERR_INVALID_ARGUMENT;
  }
  if (ws_bytes < hs.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  char* base = static_cast<char*>(ws);
  tsd_queries qd = *queries;
  qd.q = base + hs.off_q;
  int32_t* idx_d = reinterpret_cast<int32_t*>(base + hs.off_idx);
  void* out_d = base + hs.off_out;
  float* lse_d = lse != nullptr ? reinterpret_cast<float*>(base + hs.off_lse) : nullptr;
  // validate everything the decode checks before enqueueing any copy
  {
    KvView kv; QView qv; Shapes sh;
    const tsd_status st = decode_common(cache, &qd, out_d, out_dtype, lse_d, ws, dec, &kv, &qv, &sh);
    if (st != TSD_OK) return st;
  }
  const size_t lists = (size_t)queries->num_tokens * queries->num_q_heads;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(base + hs.off_q, queries->q, lists * kHeadDim * (queries->q_dtype == TSD_F32 ? 4 : 2),
                                  cudaMemcpyDefault, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(idx_d, idx, lists * (size_t)k_max * sizeof(int32_t), cudaMemcpyDefault, s);
  if (e != cudaSuccess) return TSD_ERR_CUDA;
  const tsd_status st = sparse_decode_impl(cache, &qd, idx_d, nullptr, k_max, out_d, out_dtype, lse_d, ws, dec, stream);
  if (st != TSD_OK) return st;
  e = cudaMemcpyAsync(out, out_d, lists * kHeadDim * (out_dtype == TSD_F32 ? 4 : 2), cudaMemcpyDefault, s);
  if (e == cudaSuccess && lse != nullptr) e = cudaMemcpyAsync(lse, lse_d, lists * sizeof(float), cudaMemcpyDefault, s);
  return e == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

tsd_status tsd_sparse_decode_weighted(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                      const float* logw, int32_t k_max, void* out, int32_t out_dtype, float* lse,
                                      void* ws, size_t ws_bytes, tsd_stream_t stream) {
  if (logw == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  return sparse_decode_impl(cache, queries, idx, logw, k_max, out, out_dtype, lse, ws, ws_bytes, stream);
}

tsd_status tsd_stochastic_select(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* topk_idx,
                                 int32_t k_max, const uint32_t* u, int32_t m, int32_t* out_idx, float* out_logw,
                                 uint32_t* status, tsd_stream_t stream) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = check_inputs(cache, queries, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  if (topk_idx == nullptr || out_idx == nullptr || out_logw == nullptr || k_max < 1 || m < 0) return TSD_ERR_INVALID_ARGUMENT;
  if (m > 1024) return TSD_ERR_UNSUPPORTED;
  if (m > 0 && u == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_stochastic_select(kv, qv, topk_idx, k_max, u, m, out_idx, out_logw, status,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_dense_decode(const tsd_kv_cache* cache, const tsd_queries* queries, void* out, int32_t out_dtype,
                            float* lse, void* ws, size_t ws_bytes, tsd_stream_t stream) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = decode_common(cache, queries, out, out_dtype, lse, ws, ws_bytes, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  const DensePlan p = plan_dense(sh, (int64_t)current_sm_count() * kDnCtasPerSm);
  const DecodeLayout lay = decode_layout(sh, p.nsplit);
  if (ws_bytes < lay.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.kv = kv;
  a.qv = qv;
  a.idx = nullptr;
  a.k_max = 0;
  a.span = p.window;
  a.nsplit = p.nsplit;
  a.lists_per_cta = p.lists_per_cta;
  a.list_groups = p.list_groups;
  a.out = out;
  a.out_f32 = out_dtype == TSD_F32;
  a.lse = lse;
  a.status = static_cast<uint32_t*>(ws);
  a.counters = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + lay.off_counters);
  a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + lay.off_ml);
  a.part_acc = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_acc);
  KvMaps maps;
  st = make_kv_maps(cache, &maps);
  if (st != TSD_OK) return st;
  return cuda_status(launch_dense_decode(a, maps, (int)sh.batch, (int)sh.hkv, reinterpret_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// Label-channel approximate indexer
// ---------------------------------------------------------------------------
static bool label_r_ok(int32_t r) { return r == 8 || r == 16 || r == 32; }

// The cache descriptor alone, validated through check_inputs with a stand-in query set.
static tsd_status check_cache_only(const tsd_kv_cache* cache, KvView* kv, Shapes* sh) {
  if (cache == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  tsd_queries q;
  memset(&q, 0, sizeof(q));
  q.q = cache->k;
  q.q_dtype = TSD_BF16;
  q.num_q_heads = cache->num_kv_heads;
  q.num_tokens = cache->batch;
  q.sm_scale = 1.f;
  QView qv;
  return check_inputs(cache, &q, kv, &qv, sh);
}

static int64_t cache_rows(const tsd_kv_cache* c) {
  return c->layout == TSD_LAYOUT_CONTIGUOUS ? (int64_t)c->batch * c->num_kv_heads * c->max_seq_len
                                            : c->num_pages * c->num_kv_heads * c->page_size;
}

size_t tsd_label_cache_bytes(const tsd_kv_cache* cache, int32_t r) {
  KvView kv; Shapes sh;
  if (!label_r_ok(r)) return 0;
  tsd_kv_cache c;
  if (cache == nullptr) return 0;
  c = *cache;
  static const uint16_t dummy[8] = {0};
  if (c.k == nullptr) c.k = dummy;
  if (c.v == nullptr) c.v = dummy;
  if (c.seq_lens == nullptr) c.seq_lens = reinterpret_cast<const int32_t*>(dummy);
  if (c.layout == TSD_LAYOUT_PAGED && c.page_table == nullptr) c.page_table = reinterpret_cast<const int32_t*>(dummy);
  if (check_cache_only(&c, &kv, &sh) != TSD_OK) return 0;
  return (size_t)cache_rows(&c) * r * sizeof(uint16_t);
}

size_t tsd_label_channels_workspace_size(const tsd_kv_cache* cache, const tsd_queries* queries) {
  Shapes sh;
  if (sizes_for(cache, queries, &sh) != TSD_OK) return 0;
  return label_channels_ws_bytes(sh.batch, sh.hkv);
}

tsd_status tsd_label_channels(const tsd_kv_cache* cache, const tsd_queries* queries, int32_t r, int32_t* channels,
                              void* ws, size_t ws_bytes, tsd_stream_t stream) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = check_inputs(cache, queries, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  if (!label_r_ok(r) || channels == nullptr || ws == nullptr || ((uintptr_t)ws & 255) != 0)
    return TSD_ERR_INVALID_ARGUMENT;
  if (ws_bytes < label_channels_ws_bytes(sh.batch, sh.hkv)) return TSD_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(launch_label_channels(kv, qv, r, channels, ws, reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_label_cache_build(const tsd_kv_cache* cache, const int32_t* channels, int32_t r, void* label_k,
                                 uint32_t* status, tsd_stream_t stream) {
  KvView kv; Shapes sh;
  tsd_status st = check_cache_only(cache, &kv, &sh);
  if (st != TSD_OK) return st;
  if (!label_r_ok(r)) return TSD_ERR_UNSUPPORTED;
  if (channels == nullptr || label_k == nullptr || ((uintptr_t)label_k & 15) != 0) return TSD_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_label_build(kv, channels, r, cache_rows(cache), static_cast<uint16_t*>(label_k), status,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_topk_select_label(const tsd_kv_cache* cache, const void* label_k, const int32_t* channels, int32_t r,
                                 const tsd_queries* queries, int32_t k_max, const int32_t* k_per_token,
                                 int32_t* out_idx, int32_t* out_count, void* ws, size_t ws_bytes,
                                 tsd_stream_t stream) {
  KvView kv; QView qv; Shapes sh;
  tsd_status st = check_inputs(cache, queries, &kv, &qv, &sh);
  if (st != TSD_OK) return st;
  if (!label_r_ok(r)) return TSD_ERR_UNSUPPORTED;
  if (k_max < 1 || out_idx == nullptr || ws == nullptr || label_k == nullptr || channels == nullptr)
    return TSD_ERR_INVALID_ARGUMENT;
  if (((uintptr_t)ws & 255) != 0 || ((uintptr_t)label_k & 15) != 0) return TSD_ERR_INVALID_ARGUMENT;
  const TopkLayout lay = topk_layout_for(sh, topk_filter_space(sh, k_max));
  if (ws_bytes < lay.total) return TSD_ERR_WORKSPACE_TOO_SMALL;
  TopkArgs a;
  memset(&a, 0, sizeof(a));
  a.kv = kv;
  a.qv = qv;
  a.k_max = k_max;
  a.k_per_token = k_per_token;
  a.out_idx = out_idx;
  a.out_count = out_count;
  a.scores = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_scores);
  a.score_stride = lay.score_stride;
  a.samples = reinterpret_cast<float*>(static_cast<char*>(ws) + lay.off_samples);
  a.sample_stride = lay.sample_stride;
  a.sample_shift = lay.sample_shift;
  // The candidate filter runs here only when TSD_TOPK_FILTER forces it ("1" or "rescore"): on
  // the ragged batch at 50x it measured slower than the row form (label top-k 1779 against
  // 1200 us).  The label scores are fp32 sums over bf16 label rows whatever the query dtype.
  a.filter = filter_mode() > kFilterOff ? topk_filter_choice(sh, false, false, k_max) : 0;
  if (a.filter) a.sample_shift = lay.sample_shift + 1;
  a.cand_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 256);
  a.lo_key = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + lay.off_lo);
  a.cand = reinterpret_cast<uint2*>(static_cast<char*>(ws) + lay.off_cand);
  a.meta = reinterpret_cast<int2*>(static_cast<char*>(ws) + lay.off_meta);
  a.queue = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + lay.off_queue);
  a.queue_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 16);
  a.queue_done = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 20);
  {
    const int64_t qc = 2LL * current_sm_count();
    a.queue_ctas = (int)(qc < sh.tokens * sh.hq ? qc : sh.tokens * sh.hq);
  }
  a.label = static_cast<const uint16_t*>(label_k);
  a.channels = channels;
  a.label_r = r;
  const DensePlan p = plan_dense(sh, (int64_t)current_sm_count() * kDnCtasPerSm, kMaxWindowScore);
  a.lists_per_cta = p.lists_per_cta;
  a.list_groups = p.list_groups;
  a.window = p.window;
  a.status = static_cast<uint32_t*>(ws);
  return cuda_status(launch_label_topk(a, static_cast<const uint16_t*>(label_k), channels, r, p.nsplit,
                                       (int)sh.batch, (int)sh.hkv, (int)(sh.tokens * sh.hq),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

tsd_status tsd_read_device_status(void* ws, tsd_stream_t stream, uint32_t* flags) {
  if (ws == nullptr || flags == nullptr) return TSD_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return TSD_ERR_CUDA;
  *flags = host;
  return host ? TSD_ERR_DEVICE_STATUS : TSD_OK;
}

}  // extern "C"

namespace tsd {

// Validation and argument setup for tsd_sparse_decode_static_ws (tsd_static_ws.cu): the
// same checks and work decomposition as tsd_sparse_decode, minus the workspace pointers,
// plus the bytes the layout needs (`ws_needed`) and the size of its zero region.
tsd_status prepare_sparse_decode(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                 int32_t k_max, void* out, int32_t out_dtype, float* lse, DecodeArgs* a,
                                 Shapes* sh, size_t* ws_needed, size_t* zero_bytes) {
  KvView kv; QView qv;
  tsd_status st = check_inputs(cache, queries, &kv, &qv, sh);
  if (st != TSD_OK) return st;
  if (out == nullptr || idx == nullptr || k_max < 1) return TSD_ERR_INVALID_ARGUMENT;
  if (out_dtype != TSD_BF16 && out_dtype != TSD_F32) return TSD_ERR_UNSUPPORTED;
  if (k_max > kMaxSparseK) return TSD_ERR_UNSUPPORTED;
  const SparsePlan p = sparse_plan(*sh, k_max);
  const DecodeLayout lay = decode_layout(*sh, p.nsplit);
  memset(a, 0, sizeof(*a));
  a->persistent = p.stream;
  a->kv = kv;
  a->qv = qv;
  a->idx = idx;
  a->k_max = k_max;
  a->span = p.entries;
  a->nsplit = p.nsplit;
  a->lists_per_cta = p.lists;
  a->list_groups = 1;
  a->out = out;
  a->out_f32 = out_dtype == TSD_F32;
  a->lse = lse;
  *ws_needed = lay.total;
  *zero_bytes = zero_region_bytes(*sh);
  return TSD_OK;
}

}  // namespace tsd
