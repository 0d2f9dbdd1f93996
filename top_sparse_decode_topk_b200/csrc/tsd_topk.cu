// Exact top-k token selection ("Oracle Top-K") for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?",
// gist.science summary, section 2): for every query token t and q head h keep
// the k tokens with the largest q.K, exactly; ties go to the lower token index
// and the kept indices are written in ascending order.
//
// Two kernels:
//  * topk_score_kernel -- one CTA per (sequence, kv head, list group, 1024-token
//    window).  K rows stream through a 4-stage cp.async ring of 32-row tiles;
//    each row is read from HBM once and scored against every query of the GQA
//    group and every decode token of the sequence (up to 32 lists per CTA).
//    Lane-groups of 8 lanes hold 4 query vectors (16 dims per lane) and reduce
//    the 4 dots with a 4-shuffle transposed butterfly.  Scores are fp32
//    (bf16 x bf16 products are exact in fp32; only the sum rounds).
//  * topk_select_kernel -- one CTA per (t, h).  Scores map to order-preserving
//    uint32 keys; an 11-bit histogram finds the bin holding the k-th key,
//    further digit passes narrow it until the candidates fit shared memory, a
//    radix select over the candidates gives the exact k-th key T, and a final
//    ordered pass keeps every key > T plus the lowest-index keys == T, writing
//    them in ascending token order with block-wide prefix sums.
#include <cuda_runtime.h>
#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"

namespace tsd {

constexpr int kScoreRows = 32;                   // rows per tile
constexpr int kScoreStages = 4;
constexpr int kScoreTileBytes = kScoreRows * 256;
constexpr int kHeadsPerScoreGroup = 4;
constexpr int kSelBins = 2048;
constexpr int kCandMax = 8192;
constexpr int kSelPerThread = 16;                 // scores per thread per tile (4 x float4)


// ---------------------------------------------------------------------------
// Scoring
// ---------------------------------------------------------------------------
struct ScoreSmem {
  unsigned char ring[kScoreStages * kScoreTileBytes];
  uint32_t rowaddr[kScoreStages][kScoreRows];
};

__device__ __forceinline__ void score_load_tile(ScoreSmem& S, const KvView& kv, int b, int g, int tok0,
                                                int tile, int ntok, uint32_t* status) {
  const int stage = tile % kScoreStages;
  unsigned char* base = S.ring + stage * kScoreTileBytes;
  const int first = tok0 + tile * kScoreRows;
#pragma unroll
  for (int q = 0; q < (kScoreRows * 16) / kScoreThreads; ++q) {
    const int id = threadIdx.x + q * kScoreThreads;
    const int r = id >> 4, ch = id & 15;
    const int tok = first + r;
    if (tok - tok0 < ntok) {
      const uint32_t row = kv_row(kv, b, g, tok);
      if (row != kInvalidRow) cp_async16(base + r * 256 + ch * 16, kv.k + (int64_t)row * kHeadDim + ch * 8);
      if (ch == 0) {
        S.rowaddr[stage][r] = row;
        if (row == kInvalidRow) flag_status(status, TSD_DEV_BAD_PAGE);
      }
    }
  }
}

__global__ void __launch_bounds__(kScoreThreads, 2) topk_score_kernel(TopkArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  ScoreSmem& S = *reinterpret_cast<ScoreSmem*>(smem_raw);
  const int win = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, win == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;
  const int tok0 = win * a.window;
  int ntok = si.len - tok0;
  if (ntok > a.window) ntok = a.window;
  if (ntok <= 0) return;
  const int ntiles = (ntok + kScoreRows - 1) / kScoreRows;

#pragma unroll
  for (int s = 0; s < kScoreStages - 1; ++s) {
    if (s < ntiles) score_load_tile(S, a.kv, b, g, tok0, s, ntok, a.status);
    cp_async_commit();
  }

  const int group = threadIdx.x >> 3, l8 = threadIdx.x & 7;
  const int nsets = (nlists + kHeadsPerScoreGroup - 1) / kHeadsPerScoreGroup;   // <= 8
  const int PG = 32 / nsets;
  const int my_set = group / PG, my_part = group % PG;
  const bool has_set = my_set < nsets;

  // the 4 query vectors of this group's set; lane l8 holds dims [8*l8, +8) and [64+8*l8, +8)
  float q[kHeadsPerScoreGroup][16];
  int kvlen[kHeadsPerScoreGroup];
  int64_t srow[kHeadsPerScoreGroup];
#pragma unroll
  for (int hh = 0; hh < kHeadsPerScoreGroup; ++hh) {
    const int m = my_set * kHeadsPerScoreGroup + hh;
    const bool ok = has_set && m < nlists;
    const int mg = lg * a.lists_per_cta + (ok ? m : 0);
    const int j = mg / G;
    const int t = si.t0 + j, h = g * G + (mg - j * G);
    kvlen[hh] = ok ? kv_len_of(a.qv, si, j) : 0;
    srow[hh] = ((int64_t)t * a.qv.hq + h) * a.score_stride;
    const int64_t base = ((int64_t)t * a.qv.hq + h) * kHeadDim;
    if (a.qv.q_f32) {
      const float* p = reinterpret_cast<const float*>(a.qv.q) + base;
#pragma unroll
      for (int j2 = 0; j2 < 8; ++j2) {
        q[hh][j2] = __ldg(p + 8 * l8 + j2);
        q[hh][8 + j2] = __ldg(p + 64 + 8 * l8 + j2);
      }
    } else {
      const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.qv.q) + base);
      unpack8(__ldg(p + l8), q[hh]);
      unpack8(__ldg(p + 8 + l8), q[hh] + 8);
    }
  }
  // after the transposed reduction lane l8 holds the dot of head ((l8>>2)&1)*2 + ((l8>>1)&1)
  const int my_head = ((l8 >> 2) & 1) * 2 + ((l8 >> 1) & 1);
  int my_kvlen = kvlen[0];
  int64_t my_srow = srow[0];
#pragma unroll
  for (int hh = 1; hh < kHeadsPerScoreGroup; ++hh)
    if (my_head == hh) { my_kvlen = kvlen[hh]; my_srow = srow[hh]; }

  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<kScoreStages - 2>();
    __syncthreads();
    if (tile + kScoreStages - 1 < ntiles) score_load_tile(S, a.kv, b, g, tok0, tile + kScoreStages - 1, ntok, a.status);
    cp_async_commit();
    const int stage = tile % kScoreStages;
    const unsigned char* kbase = S.ring + stage * kScoreTileBytes;
    const int rows = min(kScoreRows, ntok - tile * kScoreRows);
    for (int r0 = 0; r0 < kScoreRows; r0 += PG) {
      const int r = r0 + my_part;
      const int rr = r < kScoreRows ? r : 0;
      const unsigned char* krow = kbase + rr * 256;
      uint4 k0 = *reinterpret_cast<const uint4*>(krow + 16 * l8);
      uint4 k1 = *reinterpret_cast<const uint4*>(krow + 128 + 16 * l8);
      float kf[16];
      unpack8(k0, kf);
      unpack8(k1, kf + 8);
      float v[kHeadsPerScoreGroup];
#pragma unroll
      for (int hh = 0; hh < kHeadsPerScoreGroup; ++hh) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          s0 = fmaf(q[hh][j], kf[j], s0);
          s1 = fmaf(q[hh][8 + j], kf[8 + j], s1);
        }
        v[hh] = s0 + s1;
      }
      // transposed butterfly: 4 partial dots over 8 lanes -> one full dot per lane pair
      const bool hi4 = (l8 & 4) != 0;
      float a0 = hi4 ? v[2] : v[0], a1 = hi4 ? v[3] : v[1];
      float s0 = hi4 ? v[0] : v[2], s1 = hi4 ? v[1] : v[3];
      a0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 4);
      a1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 4);
      const bool hi2 = (l8 & 2) != 0;
      float c = hi2 ? a1 : a0, d = hi2 ? a0 : a1;
      c += __shfl_xor_sync(0xFFFFFFFFu, d, 2);
      c += __shfl_xor_sync(0xFFFFFFFFu, c, 1);
      const int tok = tok0 + tile * kScoreRows + rr;
      const bool ok = has_set && r < rows && (l8 & 1) == 0 && tok < my_kvlen &&
                      S.rowaddr[stage][rr] != kInvalidRow;
      if (ok) a.scores[my_srow + tok] = c;
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Selection
// ---------------------------------------------------------------------------
struct SelectSmem {
  uint32_t hist[kSelBins];
  uint32_t cand[kCandMax];
  int scan_tmp[kSelectThreads / 32 + 1];
  int found_bin, found_above, ncand;
};

// hist[0..nbins): find d with count(> d) < need <= count(>= d).  Results in S.found_*.
__device__ void select_bin(SelectSmem& S, int nbins, int need) {
  if (threadIdx.x == 0) {   // defined result even if no bin qualifies (cannot happen for consistent data)
    S.found_bin = 0;
    S.found_above = 0;
  }
  const int per = (nbins + kSelectThreads - 1) / kSelectThreads;
  const int hi = nbins - threadIdx.x * per;     // this thread owns bins [hi-per, hi) from the top
  int local = 0;
  for (int j = 0; j < per; ++j) {
    const int bin = hi - 1 - j;
    if (bin >= 0) local += (int)S.hist[bin];
  }
  int total;
  int run = block_exclusive_scan<kSelectThreads>(local, S.scan_tmp, &total);
  for (int j = 0; j < per; ++j) {
    const int bin = hi - 1 - j;
    if (bin < 0) break;
    const int c = (int)S.hist[bin];
    if (run < need && run + c >= need) {
      S.found_bin = bin;
      S.found_above = run;
    }
    run += c;
  }
  __syncthreads();
}

__device__ __forceinline__ void load16(const float* row, int i0, int L, float* f) {
  // 16 consecutive scores from i0 (i0 multiple of 4); beyond L the values are unused
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = i0 + 4 * j;
    float4 v = (i < L) ? __ldcg(reinterpret_cast<const float4*>(row + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    f[4 * j] = v.x; f[4 * j + 1] = v.y; f[4 * j + 2] = v.z; f[4 * j + 3] = v.w;
  }
}

__global__ void __launch_bounds__(kSelectThreads, 2) topk_select_kernel(TopkArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelectSmem& S = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int th = blockIdx.x;
  const int t = th / a.qv.hq;

  // sequence of token t
  int b;
  if (a.qv.q_indptr == nullptr) {
    b = t;
  } else {
    int lo = 0, hi = a.kv.batch;   // largest b with q_indptr[b] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.qv.q_indptr + mid) <= t) lo = mid; else hi = mid;
    }
    b = lo;
  }
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, false);
  int L = 0;
  if (t >= si.t0 && t < si.t0 + si.n) L = kv_len_of(a.qv, si, t - si.t0);
  int kreq = a.k_max;
  if (a.k_per_token != nullptr) {
    kreq = __ldg(a.k_per_token + t);
    kreq = kreq < 0 ? 0 : (kreq > a.k_max ? a.k_max : kreq);
  }
  const int k = kreq < L ? kreq : L;
  int32_t* out = a.out_idx + (int64_t)th * a.k_max;
  if (a.out_count != nullptr && threadIdx.x == 0) a.out_count[th] = k;

  if (k == L) {   // every visible token is kept (covers k == 0 with L == 0)
    for (int i = threadIdx.x; i < a.k_max; i += kSelectThreads) out[i] = i < L ? i : -1;
    return;
  }
  const float* row = a.scores + (int64_t)th * a.score_stride;
  const int tile_elems = kSelectThreads * kSelPerThread;

  // ---- pass 1: histogram of the top 11 key bits ----
  for (int i = threadIdx.x; i < kSelBins; i += kSelectThreads) S.hist[i] = 0u;
  __syncthreads();
  for (int base = 0; base < L; base += tile_elems) {
    const int i0 = base + threadIdx.x * kSelPerThread;
    float f[kSelPerThread];
    load16(row, i0, L, f);
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j)
      if (i0 + j < L) atomicAdd(&S.hist[score_key(f[j]) >> 21], 1u);
  }
  __syncthreads();
  select_bin(S, kSelBins, k);
  uint32_t prefix = (uint32_t)S.found_bin & (kSelBins - 1);
  int need = k - S.found_above;
  int ccount = (int)S.hist[prefix];
  int shift = 21;
  __syncthreads();

  // ---- refinement passes over global memory while the candidates do not fit ----
  while (ccount > kCandMax && shift > 0) {
    const int nb = shift >= 11 ? 11 : shift;
    shift -= nb;
    for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[i] = 0u;
    __syncthreads();
    for (int base = 0; base < L; base += tile_elems) {
      const int i0 = base + threadIdx.x * kSelPerThread;
      float f[kSelPerThread];
      load16(row, i0, L, f);
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j) {
        const uint32_t key = score_key(f[j]);
        if (i0 + j < L && (key >> (shift + nb)) == prefix) atomicAdd(&S.hist[(key >> shift) & ((1u << nb) - 1)], 1u);
      }
    }
    __syncthreads();
    select_bin(S, 1 << nb, need);
    const uint32_t d = (uint32_t)S.found_bin & ((1u << nb) - 1);
    prefix = (prefix << nb) | d;
    need -= S.found_above;
    ccount = (int)S.hist[d];
    __syncthreads();
  }

  // ---- candidates into shared memory, then radix select among them ----
  if (shift > 0) {
    if (threadIdx.x == 0) S.ncand = 0;
    __syncthreads();
    for (int base = 0; base < L; base += tile_elems) {
      const int i0 = base + threadIdx.x * kSelPerThread;
      float f[kSelPerThread];
      load16(row, i0, L, f);
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j) {
        const uint32_t key = score_key(f[j]);
        if (i0 + j < L && (key >> shift) == prefix) {
          const int pos = atomicAdd(&S.ncand, 1);
          if (pos < kCandMax) S.cand[pos] = key;
        }
      }
    }
    __syncthreads();
    const int nc = S.ncand < kCandMax ? S.ncand : kCandMax;
    while (shift > 0) {
      const int nb = shift >= 8 ? 8 : shift;
      shift -= nb;
      for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[i] = 0u;
      __syncthreads();
      for (int c = threadIdx.x; c < nc; c += kSelectThreads) {
        const uint32_t key = S.cand[c];
        if ((key >> (shift + nb)) == prefix) atomicAdd(&S.hist[(key >> shift) & ((1u << nb) - 1)], 1u);
      }
      __syncthreads();
      select_bin(S, 1 << nb, need);
      prefix = (prefix << nb) | ((uint32_t)S.found_bin & ((1u << nb) - 1));
      need -= S.found_above;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;   // the exact k-th largest key
  const int need_eq = need;    // how many keys == T are kept (the lowest indices)

  // ---- output pass: ordered compaction of (key > T) or (key == T and among the first need_eq) ----
  int eq_before = 0, sel_before = 0;
  for (int base = 0; base < L; base += tile_elems) {
    const int i0 = base + threadIdx.x * kSelPerThread;
    float f[kSelPerThread];
    load16(row, i0, L, f);
    uint32_t keys[kSelPerThread];
    int neq = 0;
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j) {
      keys[j] = score_key(f[j]);
      if (i0 + j < L && keys[j] == T) ++neq;
    }
    int eq_total;
    int eq_run = eq_before + block_exclusive_scan<kSelectThreads>(neq, S.scan_tmp, &eq_total);
    int nsel = 0;
    uint32_t selmask = 0;
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j) {
      bool sel = false;
      if (i0 + j < L) {
        if (keys[j] > T) sel = true;
        else if (keys[j] == T) { sel = eq_run < need_eq; ++eq_run; }
      }
      if (sel) { selmask |= 1u << j; ++nsel; }
    }
    int sel_total;
    int pos = sel_before + block_exclusive_scan<kSelectThreads>(nsel, S.scan_tmp, &sel_total);
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j)
      if (selmask & (1u << j)) {
        if (pos < k) out[pos] = i0 + j;
        ++pos;
      }
    eq_before += eq_total;
    sel_before += sel_total;
  }
  for (int i = k + threadIdx.x; i < a.k_max; i += kSelectThreads) out[i] = -1;
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_topk(const TopkArgs& a, int nwin, int batch, int hkv, int num_lists, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(ScoreSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SelectSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 g1(nwin, hkv * a.list_groups, batch);
  topk_score_kernel<<<g1, kScoreThreads, sizeof(ScoreSmem), stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<num_lists, kSelectThreads, sizeof(SelectSmem), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tsd
