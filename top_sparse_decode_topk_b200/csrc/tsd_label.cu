// Label-channel approximate indexer (Double-Sparsity-style) for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?", gist.science
// summary, section 3.C, indexing overhead): the pages price the indexer in front of sparse
// decode with Double Sparsity -- every token is scored with only a few "label" channels of
// its key, kept in a compact cache, and the top k of those approximate scores are kept.
// The channel count and choice are not on the pages; here r channels per kv head with the
// largest total |q_d K_{i,d}| over the calibration pairs (ties to the lower channel), and
// the top-k of s~_i = sum over the label channels of q_d K_{i,d}.
//
// Kernels:
//  * label_ksum_kernel    -- per (sequence, kv head, token split): sums of |K[., d]| (fp32
//                            per thread, a fixed reduction order: deterministic).
//  * label_choose_kernel  -- per kv head: importance_d = sum_b (sum_{t in b, h in g} |q_{t,h,d}|)
//                            x (sum_i |K_{b,g,i,d}|) in fp64, then the r largest, ascending.
//  * label_build_kernel   -- gathers the label channels of every cache row into the compact
//                            label cache (same row numbering as K, r bf16 per row).
//  * label_score_kernel<R> -- per (sequence, kv head, list group, token window): reads the
//                            2R-byte label rows once for every list of the GQA group and writes
//                            fp32 approximate scores; the exact select kernel then picks top-k.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"
#include "tsd_filter.cuh"

namespace tsd {

constexpr int kLblSplits = 16;       // token splits per (sequence, kv head) for the |K| sums
constexpr int kLblThreads = 256;
constexpr int kLblUnroll = 4;        // tokens per thread in flight in the scoring kernel

// ---------------------------------------------------------------------------
// Channel choice (offline calibration)
// ---------------------------------------------------------------------------
// partial[((b * hkv + g) * kLblSplits + s) * 128 + d] = sum over this split's tokens of |K|.
__global__ void __launch_bounds__(kLblThreads) label_ksum_kernel(KvView kv, float* partial, uint32_t* status) {
  __shared__ float red[kLblThreads / 16][kHeadDim];
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int l = threadIdx.x & 15, rgrp = threadIdx.x >> 4;   // 16 row groups x 16 lanes of 8 dims
  int len = __ldg(kv.seq_lens + b);
  if (len < 0 || len > kv.max_seq_len) {
    if (threadIdx.x == 0 && s == 0 && g == 0) flag_status(status, TSD_DEV_BAD_SEQ);
    len = 0;
  }
  const int per = (len + kLblSplits - 1) / kLblSplits;
  const int i0 = s * per, i1 = min(len, i0 + per);
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int i = i0 + rgrp; i < i1; i += kLblThreads / 16) {
    const uint32_t row = kv_row(kv, b, g, i);
    if (row == kInvalidRow) {
      if (l == 0) flag_status(status, TSD_DEV_BAD_PAGE);
      continue;
    }
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(kv.k + (int64_t)row * kHeadDim) + l), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += fabsf(f[j]);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[rgrp][8 * l + j] = acc[j];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    float t = 0.f;
    for (int r = 0; r < kLblThreads / 16; ++r) t += red[r][threadIdx.x];
    partial[(((int64_t)b * kv.hkv + g) * kLblSplits + s) * kHeadDim + threadIdx.x] = t;
  }
}

// One CTA of 128 threads (thread d = channel d) per kv head g.
__global__ void __launch_bounds__(kHeadDim) label_choose_kernel(KvView kv, QView qv, const float* partial, int r,
                                                                int32_t* channels) {
  __shared__ double imp[kHeadDim];
  __shared__ int warp_sel[kHeadDim / 32];
  const int g = blockIdx.x, d = threadIdx.x;
  const int G = qv.hq / kv.hkv;
  double total = 0.0;
  for (int b = 0; b < kv.batch; ++b) {
    int t0 = b, t1 = b + 1;
    if (qv.q_indptr != nullptr) {
      t0 = __ldg(qv.q_indptr + b);
      t1 = __ldg(qv.q_indptr + b + 1);
    }
    t0 = max(0, t0);
    t1 = min(t1, qv.num_tokens);
    double qs = 0.0;
    for (int t = t0; t < t1; ++t)
      for (int h = g * G; h < (g + 1) * G; ++h) {
        const int64_t e = ((int64_t)t * qv.hq + h) * kHeadDim + d;
        const float x = qv.q_f32 ? __ldg(reinterpret_cast<const float*>(qv.q) + e)
                                 : __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(qv.q) + e) << 16);
        qs += fabs((double)x);
      }
    double ks = 0.0;
    for (int s = 0; s < kLblSplits; ++s) ks += (double)partial[(((int64_t)b * kv.hkv + g) * kLblSplits + s) * kHeadDim + d];
    total += qs * ks;
  }
  imp[d] = total;
  __syncthreads();
  int rank = 0;   // channels ahead of d: larger importance, or equal with a lower index
  for (int e = 0; e < kHeadDim; ++e) rank += (imp[e] > total) || (imp[e] == total && e < d);
  const bool sel = rank < r;
  const unsigned ball = __ballot_sync(0xFFFFFFFFu, sel);
  if ((d & 31) == 0) warp_sel[d >> 5] = __popc(ball);
  __syncthreads();
  int pos = __popc(ball & ((1u << (d & 31)) - 1u));
  for (int w = 0; w < (d >> 5); ++w) pos += warp_sel[w];
  if (sel) channels[(int64_t)g * r + pos] = d;
}

// ---------------------------------------------------------------------------
// Label cache: out[row * r + j] = K[row * 128 + channels[g(row) * r + j]]
// ---------------------------------------------------------------------------
__global__ void label_build_kernel(KvView kv, const int32_t* channels, int r, int64_t rows, uint16_t* label,
                                   uint32_t* status) {
  const int64_t n = rows * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / r;
    const int j = (int)(e - row * r);
    const int g = kv.page_table != nullptr ? (int)((row >> kv.page_shift) % kv.hkv)
                                           : (int)((row / kv.max_seq_len) % kv.hkv);
    int c = __ldg(channels + (int64_t)g * r + j);
    if (c < 0 || c >= kHeadDim) {
      if (status != nullptr) flag_status(status, TSD_DEV_BAD_INDEX);
      c = 0;
    }
    label[e] = __ldg(kv.k + row * kHeadDim + c);
  }
}

// ---------------------------------------------------------------------------
// Approximate scores
// ---------------------------------------------------------------------------
// One CTA per (window, kv head x list group, sequence); each thread scores tokens
// tok0 + threadIdx.x, + 256, ... against up to 16 lists whose label queries sit in shared
// memory.  Unscaled fp32 dots; bf16 x bf16 products are exact, only the R-term sum rounds.
// NL = 0: any number of lists (at most 16), their queries, bounds and score rows read from shared
// memory per list.  NL = 4: at most 4 lists (one decode token of a GQA group of 4, as in the
// Llama-3-8B shape), whose query pairs, bounds and score rows live in registers, the list loop
// unrolled; 2 tokens per lane per step keep the registers within two CTAs per SM.
// ---------------------------------------------------------------------------
// Candidate filter of the label indexer (as the exact indexer's, in tsd_topk.cu)
// ---------------------------------------------------------------------------
// label_prepass_kernel scores every 2^sample_shift-th token of every list on the label channels
// and turns each list's sample into a threshold; label_score_kernel then appends the scores that
// reach it instead of writing score rows, and the exact indexer's candidate kernel and queue
// pass select from there.  A warp stages the candidates of one list and one token step in the
// CTA's shared-memory buffer with a ballot and one shared atomic; when the CTA ends, one global
// atomic per list reserves the list's range and the CTA copies its candidates out.  Candidates
// that find the buffer full go straight to the list's buffer.
constexpr uint32_t kLblStage = 4096;   // staged candidates per CTA (32 KB)
constexpr uint32_t kLblStageHole = 0xFFFFFFFFu;

// Warp-collective: lanes with `cand` stage (key(sc), tok | m << 24) for list m.
__device__ __forceinline__ void stage_append(bool cand, float sc, uint32_t tok, int m, uint2* st, uint32_t* nst,
                                             uint32_t* lcnt, uint32_t* gcnt, uint2* gbuf, int lane) {
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
  if (bal == 0u) return;
  const uint32_t n = __popc(bal);
  uint32_t base = 0u;
  if (lane == 0) base = atomicAdd(nst, n);
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  const uint32_t i = __popc(bal & ((1u << lane) - 1u));
  if (base + n <= kLblStage) {
    if (cand) st[base + i] = make_uint2(score_key(sc), tok | ((uint32_t)m << 24));
    if (lane == 0) atomicAdd(lcnt + m, n);
    return;
  }
  // the buffer is full: the slots this call took inside it become holes, the candidates go out
  if (cand && base + i < kLblStage) st[base + i] = make_uint2(0u, kLblStageHole);
  uint32_t g = 0u;
  if (lane == 0) g = atomicAdd(gcnt, n);
  g = __shfl_sync(0xFFFFFFFFu, g, 0);
  if (cand && g + i < (uint32_t)kTopkCandCap) gbuf[g + i] = make_uint2(score_key(sc), tok);
}

// Grid (Hkv x list groups, batch), kLblThreads threads: thread i scores samples i, i + 256, ...
// of the group's lists, then warp w makes the thresholds of lists w, w + 8, ...
template <int R>
__global__ void __launch_bounds__(kLblThreads) label_prepass_kernel(TopkArgs a) {
  __shared__ float qs[16][R];
  const int g = blockIdx.x / a.list_groups, lg = blockIdx.x % a.list_groups;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();   // the scoring kernel may launch; it waits for this grid
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, false);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;
  for (int e = threadIdx.x; e < 16 * R; e += kLblThreads) {
    const int m = e / R, j = e - (e / R) * R;
    float v = 0.f;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int jt = mg / G;
      int c = __ldg(a.channels + (int64_t)g * R + j);
      if (c < 0 || c >= kHeadDim) c = 0;   // the scoring kernel flags it
      const int64_t qe = ((int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G)) * kHeadDim + c;
      v = a.qv.q_f32 ? __ldg(reinterpret_cast<const float*>(a.qv.q) + qe)
                     : __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(a.qv.q) + qe) << 16);
    }
    qs[m][j] = v;
  }
  __syncthreads();
  const int shift = a.sample_shift;
  const int ns_seq = (int)(((int64_t)si.len + (1 << shift) - 1) >> shift);
  for (int j = threadIdx.x; j < ns_seq; j += kLblThreads) {
    const int tok = j << shift;
    const uint32_t row = kv_row(a.kv, b, g, tok);
    if (row == kInvalidRow) continue;   // the scoring kernel flags it
    float lv[R];
    const uint4* src = reinterpret_cast<const uint4*>(a.label + (int64_t)row * R);
#pragma unroll
    for (int c = 0; c < R / 8; ++c) {
      const uint4 v = __ldg(src + c);
      lv[8 * c + 0] = bf16lo(v.x); lv[8 * c + 1] = bf16hi(v.x);
      lv[8 * c + 2] = bf16lo(v.y); lv[8 * c + 3] = bf16hi(v.y);
      lv[8 * c + 4] = bf16lo(v.z); lv[8 * c + 5] = bf16hi(v.z);
      lv[8 * c + 6] = bf16lo(v.w); lv[8 * c + 7] = bf16hi(v.w);
    }
    for (int m = 0; m < nlists; ++m) {
      const int mg = lg * a.lists_per_cta + m;
      const int jt = mg / G;
      if (tok >= kv_len_of(a.qv, si, jt)) continue;
      float sc = 0.f;
#pragma unroll
      for (int c = 0; c < R; ++c) sc = fmaf(qs[m][c], lv[c], sc);
      a.samples[((int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G)) * a.sample_stride + j] = sc;
    }
  }
  __threadfence();
  __syncthreads();
  for (int m = warp; m < nlists; m += kLblThreads / 32) {
    const int mg = lg * a.lists_per_cta + m;
    const int jt = mg / G;
    const int64_t list = (int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G);
    const int L = kv_len_of(a.qv, si, jt);
    const int k = list_k(a, si.t0 + jt, L);
    const uint32_t lo = list_threshold(a.samples + list * a.sample_stride, L, k, shift, a.filter == 1, lane);
    if (lane == 0) {
      a.lo_key[list] = lo;
      a.meta[list] = make_int2(L, k);
    }
  }
}

// resident CTAs per SM: the row form's counts as measured (r = 8 with many lists in 64 registers,
// r = 16 with many lists in 80, the rest in 128); the filtered form, with its 34 KB of staged
// candidates, two
constexpr int label_score_min_ctas(int R, int NL, bool filt) {
  return filt ? 2 : (NL == 0 && R == 8 ? 4 : (NL == 0 && R == 16 ? 3 : 2));
}
template <int R, int NL, bool FILT>
__global__ void __launch_bounds__(kLblThreads, label_score_min_ctas(R, NL, FILT)) label_score_kernel(TopkArgs a, const uint16_t* label,
                                                                  const int32_t* channels) {
  // FILT: the filtered form, instantiated apart so that the row form keeps its registers
  __shared__ __align__(16) float qs[16][R];
  __shared__ int kvl[16];
  __shared__ int64_t srow[16];
  __shared__ int64_t prow[16];   // the list's sample row (every 2^sample_shift-th token's score)
  const int win = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, win == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  const int tok0 = win * a.window;
  const int tok_end = min(tok0 + a.window, si.len);
  if (nlists <= 0 || tok_end <= tok0) {
    // under the filter the kernels after this one read what the pre-pass wrote once this grid
    // has completed, so every CTA waits for the pre-pass before it exits
    if (FILT) pdl_wait();
    return;
  }
  __shared__ float s_lof[16];              // filter: each list's threshold as a float
  __shared__ int64_t s_list[16];           // filter: each list's index (t Hq + h)
  __shared__ uint2 s_stage[kLblStage];     // filter: the CTA's staged candidates
  __shared__ uint32_t s_nst;               // filter: staged slots taken
  __shared__ uint32_t s_lcnt[16];          // filter: staged candidates per list, then a running index
  __shared__ uint32_t s_lbase[16];         // filter: each list's reserved range
  for (int e = threadIdx.x; e < 16 * R; e += kLblThreads) {
    const int m = e / R, j = e - (e / R) * R;
    float v = 0.f;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int jt = mg / G;
      const int h = g * G + (mg - jt * G);
      int c = __ldg(channels + (int64_t)g * R + j);
      if (c < 0 || c >= kHeadDim) {
        flag_status(a.status, TSD_DEV_BAD_INDEX);
        c = 0;
      }
      const int64_t qe = ((int64_t)(si.t0 + jt) * a.qv.hq + h) * kHeadDim + c;
      v = a.qv.q_f32 ? __ldg(reinterpret_cast<const float*>(a.qv.q) + qe)
                     : __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(a.qv.q) + qe) << 16);
      if (j == 0) {
        kvl[m] = min(kv_len_of(a.qv, si, jt), tok_end);
        srow[m] = ((int64_t)(si.t0 + jt) * a.qv.hq + h) * a.score_stride;
        prow[m] = ((int64_t)(si.t0 + jt) * a.qv.hq + h) * a.sample_stride;
      }
    }
    qs[m][j] = v;
  }
  __syncthreads();
  pdl_launch_dependents();   // the selection may launch; it waits for this kernel's scores
  if (FILT) {
    pdl_wait();   // the pre-pass wrote the thresholds
    if (threadIdx.x < 16) {
      const int m = threadIdx.x;
      float lf = CUDART_INF_F;
      int64_t list = 0;
      if (m < nlists) {
        const int mg = lg * a.lists_per_cta + m;
        const int jt = mg / G;
        list = (int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G);
        const uint32_t lo = __ldcg(a.lo_key + list);
        // keys above +inf's are positive NaNs, keys below -inf's negative ones
        lf = lo >= 0xFF800000u ? CUDART_INF_F : (lo <= 0x007FFFFFu ? -CUDART_INF_F : key_score(lo));
      }
      s_lof[m] = lf;
      s_list[m] = list;
      s_lcnt[m] = 0u;
    }
    if (threadIdx.x == 0) s_nst = 0u;
    __syncthreads();
  }
  // Each warp walks steps of kLblStep consecutive tokens (lane l takes tokens 32 u + l of the
  // step), the CTA's warps taking consecutive steps.  With pages of 4 tokens or more, a step's
  // tokens lie in at most 32 pages: lane l holds the page-table entry of the step's l-th page,
  // loaded one step ahead, and every token finds its row with a shuffle, so that only the
  // label-row loads wait on memory inside a step.
  constexpr unsigned FULL = 0xFFFFFFFFu;
  constexpr int kWarps = kLblThreads / 32;
  constexpr int U = NL > 0 ? 2 : kLblUnroll;   // tokens per lane per step
  constexpr int kLblStep = 32 * U;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NR = NL > 0 ? NL : 1;
  unsigned long long qr[NR][R / 2];   // NL > 0: list m's query channel pairs
  int kvr[NR];
  int64_t srr[NR], prr[NR];
  if constexpr (NL > 0) {
#pragma unroll
    for (int m = 0; m < NL; ++m) {
      const ulonglong2* qm = reinterpret_cast<const ulonglong2*>(qs[m]);
#pragma unroll
      for (int j = 0; j < R / 4; ++j) {
        const ulonglong2 qq = qm[j];
        qr[m][2 * j] = qq.x;
        qr[m][2 * j + 1] = qq.y;
      }
      kvr[m] = m < nlists ? kvl[m] : 0;
      srr[m] = m < nlists ? srow[m] : 0;
      prr[m] = m < nlists ? prow[m] : 0;
    }
  }
  float lof[NR];          // NL > 0, filter: the thresholds
#pragma unroll
  for (int m = 0; m < NR; ++m) lof[m] = FILT && NL > 0 ? s_lof[m] : CUDART_INF_F;
  const bool paged = a.kv.page_table != nullptr;
  const int shift = a.kv.page_shift;
  const int pmask = (1 << shift) - 1;
  const bool shfl_pages = paged && shift >= 2;   // a step then spans at most 32 pages
  const int32_t* pt = paged ? a.kv.page_table + (int64_t)b * a.kv.max_pages : nullptr;
  auto step_pages = [&](int st0) -> int32_t {    // lane l: the page entry of the step's l-th page
    if (!shfl_pages || st0 >= tok_end) return -1;
    const int p = (st0 >> shift) + lane;
    return p <= ((min(st0 + kLblStep, tok_end) - 1) >> shift) ? __ldg(pt + p) : -1;
  };
  int st0 = tok0 + warp * kLblStep;
  int32_t pg = step_pages(st0);
  for (; st0 < tok_end; st0 += kWarps * kLblStep) {
    const int32_t pg_next = step_pages(st0 + kWarps * kLblStep);
    uint32_t row[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tok = st0 + 32 * u + lane;
      if (shfl_pages) {
        // tokens of a step start on a multiple of min(page, 64), so rel < 32
        const int rel = ((st0 & pmask) + 32 * u + lane) >> shift;
        const int32_t page = __shfl_sync(FULL, pg, rel & 31);
        row[u] = kInvalidRow;
        if (tok < tok_end) {
          if (page >= 0 && (int64_t)page < a.kv.num_pages)
            row[u] = (uint32_t)((((int64_t)page * a.kv.hkv + g) << shift) | (tok & pmask));
          else
            flag_status(a.status, TSD_DEV_BAD_PAGE);
        }
      } else {
        row[u] = tok < tok_end ? kv_row(a.kv, b, g, tok) : kInvalidRow;
        if (tok < tok_end && row[u] == kInvalidRow) flag_status(a.status, TSD_DEV_BAD_PAGE);
      }
    }
    uint4 raw[U][R / 8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint4* src = reinterpret_cast<const uint4*>(label + (int64_t)row[u] * R);
#pragma unroll
      for (int c = 0; c < R / 8; ++c) raw[u][c] = row[u] != kInvalidRow ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tok = st0 + 32 * u + lane;
      const bool valid = row[u] != kInvalidRow;
      if (!FILT && !valid) continue;   // the filtered form's appends are warp-collective: no early out
      // channel pairs (2i, 2i + 1) as packed fp32x2: one fma.rn.f32x2 per pair, the even
      // channels summed in the low lane and the odd ones in the high lane
      unsigned long long k2[R / 2];
#pragma unroll
      for (int c = 0; c < R / 8; ++c) {
        k2[4 * c] = bf16x2_to_f32x2(raw[u][c].x);
        k2[4 * c + 1] = bf16x2_to_f32x2(raw[u][c].y);
        k2[4 * c + 2] = bf16x2_to_f32x2(raw[u][c].z);
        k2[4 * c + 3] = bf16x2_to_f32x2(raw[u][c].w);
      }
      const bool sampled = (tok & ((1 << a.sample_shift) - 1)) == 0;
      if constexpr (NL > 0) {
#pragma unroll
        for (int m = 0; m < NL; ++m) {
          unsigned long long acc = 0ull;
#pragma unroll
          for (int j = 0; j < R / 2; ++j) acc = ffma2(qr[m][j], k2[j], acc);
          const float sc = f32x2_sum(acc);
          if constexpr (FILT) {   // every lane takes part: the append is warp-collective
            const bool cand = valid && tok < kvr[m] && !(sc < lof[m]);
            stage_append(cand, sc, (uint32_t)tok, m, s_stage, &s_nst, s_lcnt, a.cand_cnt + s_list[m],
                         a.cand + s_list[m] * kTopkCandCap, lane);
          } else if (tok < kvr[m]) {   // the row form: invalid rows left above
            a.scores[srr[m] + tok] = sc;
            if (sampled) a.samples[prr[m] + (tok >> a.sample_shift)] = sc;
          }
        }
      } else {
        for (int m = 0; m < nlists; ++m) {
          const ulonglong2* qm = reinterpret_cast<const ulonglong2*>(qs[m]);   // 16-byte shared loads
          unsigned long long acc = 0ull;
#pragma unroll
          for (int j = 0; j < R / 4; ++j) {
            const ulonglong2 qq = qm[j];
            acc = ffma2(qq.x, k2[2 * j], acc);
            acc = ffma2(qq.y, k2[2 * j + 1], acc);
          }
          const float sc = f32x2_sum(acc);
          if constexpr (FILT) {
            const bool cand = valid && tok < kvl[m] && !(sc < s_lof[m]);
            stage_append(cand, sc, (uint32_t)tok, m, s_stage, &s_nst, s_lcnt, a.cand_cnt + s_list[m],
                         a.cand + s_list[m] * kTopkCandCap, lane);
          } else if (tok < kvl[m]) {
            a.scores[srow[m] + tok] = sc;
            if (sampled) a.samples[prow[m] + (tok >> a.sample_shift)] = sc;
          }
        }
      }
    }
    pg = pg_next;
  }
  if (FILT) {
    // one global atomic per list reserves its staged candidates' range; the CTA copies them out
    __syncthreads();
    if (threadIdx.x < nlists) {
      const uint32_t c = s_lcnt[threadIdx.x];
      s_lbase[threadIdx.x] = c != 0u ? atomicAdd(a.cand_cnt + s_list[threadIdx.x], c) : 0u;
      s_lcnt[threadIdx.x] = 0u;
    }
    __syncthreads();
    const uint32_t nst = s_nst < kLblStage ? s_nst : kLblStage;
    for (uint32_t e = threadIdx.x; e < nst; e += kLblThreads) {
      const uint2 v = s_stage[e];
      if (v.y == kLblStageHole) continue;
      const int m = (int)(v.y >> 24);
      const uint32_t pos = s_lbase[m] + atomicAdd(s_lcnt + m, 1u);
      if (pos < (uint32_t)kTopkCandCap) a.cand[s_list[m] * kTopkCandCap + pos] = make_uint2(v.x, v.y & 0xFFFFFFu);
    }
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
size_t label_channels_ws_bytes(int64_t batch, int64_t hkv) {
  return 256 + (size_t)batch * hkv * kLblSplits * kHeadDim * sizeof(float);
}

cudaError_t launch_label_channels(const KvView& kv, const QView& qv, int r, int32_t* channels, void* ws,
                                  cudaStream_t stream) {
  uint32_t* status = static_cast<uint32_t*>(ws);
  float* partial = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
  label_ksum_kernel<<<dim3(kLblSplits, kv.hkv, kv.batch), kLblThreads, 0, stream>>>(kv, partial, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  label_choose_kernel<<<kv.hkv, kHeadDim, 0, stream>>>(kv, qv, partial, r, channels);
  return cudaGetLastError();
}

cudaError_t launch_label_build(const KvView& kv, const int32_t* channels, int r, int64_t rows, uint16_t* label,
                               uint32_t* status, cudaStream_t stream) {
  const int64_t n = rows * r;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  label_build_kernel<<<(unsigned)blocks, 256, 0, stream>>>(kv, channels, r, rows, label, status);
  return cudaGetLastError();
}

cudaError_t launch_topk_select_only(const TopkArgs& a, int num_lists, cudaStream_t stream);
cudaError_t launch_topk_candidates(const TopkArgs& a, int num_lists, cudaStream_t stream);

cudaError_t launch_label_topk(const TopkArgs& a, const uint16_t* label, const int32_t* channels, int r, int nwin,
                              int batch, int hkv, int num_lists, cudaStream_t stream) {
  dim3 grid(nwin, hkv * a.list_groups, batch);
  const bool few = a.lists_per_cta <= 4;   // the lists' queries fit in registers (r <= 16)
  cudaError_t e = cudaSuccess;
  if (a.filter) {   // the candidate filter's pre-pass: label-score samples and thresholds
    const dim3 g0(hkv * a.list_groups, batch);
    switch (r) {
      case 8: label_prepass_kernel<8><<<g0, kLblThreads, 0, stream>>>(a); break;
      case 16: label_prepass_kernel<16><<<g0, kLblThreads, 0, stream>>>(a); break;
      case 32: label_prepass_kernel<32><<<g0, kLblThreads, 0, stream>>>(a); break;
      default: return cudaErrorInvalidValue;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // under the filter a programmatic dependent of the pre-pass, whose thresholds it waits for
  auto score = [&](auto kernel) -> cudaError_t {
    if (a.filter) return launch_dependent(kernel, grid, dim3(kLblThreads), 0, stream, a, label, channels);
    kernel<<<grid, kLblThreads, 0, stream>>>(a, label, channels);
    return cudaGetLastError();
  };
  const bool f = a.filter != 0;
  switch (r) {
    case 8:
      if (few) e = f ? score(label_score_kernel<8, 4, true>) : score(label_score_kernel<8, 4, false>);
      else e = f ? score(label_score_kernel<8, 0, true>) : score(label_score_kernel<8, 0, false>);
      break;
    case 16:
      if (few) e = f ? score(label_score_kernel<16, 4, true>) : score(label_score_kernel<16, 4, false>);
      else e = f ? score(label_score_kernel<16, 0, true>) : score(label_score_kernel<16, 0, false>);
      break;
    case 32: e = f ? score(label_score_kernel<32, 0, true>) : score(label_score_kernel<32, 0, false>); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if (a.filter) return launch_topk_candidates(a, num_lists, stream);
  return launch_topk_select_only(a, num_lists, stream);
}

}  // namespace tsd
