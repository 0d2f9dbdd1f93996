// vAttention-style stochastic selection for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?", gist.science
// summary, section 2: vAttention's stochastic index selection, evaluated against
// deterministic top-k).  The pages give no sampling scheme or estimator; here, per (query
// token t, q head h): the exact top-k list S (from tsd_topk_select), plus m tokens drawn
// uniformly without replacement from the rest R = [0, kv_len) minus S by Floyd's algorithm
// (driven by caller-supplied random 32-bit words), each weighted by |R| / m -- the
// Horvitz-Thompson estimate of the softmax sums over R.  The output is one ascending index
// list with a natural-log weight per entry (0 for S), which the weighted sparse decode
// consumes.
//
// One warp per list.  Floyd's m draws are computed in parallel; collisions are then resolved
// in step order by parallel searches for the first repeated value, one search per collision.  The kept ranks are then sorted by
// counting, mapped to tokens of R by a binary search over S (token = rank + #{s in S below it}),
// and merged with S: each sample by a binary search over S, each lane's contiguous chunk of S by
// one binary search and a forward scan of the samples.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"

namespace tsd {

constexpr int kStoMaxM = 1024;
constexpr int kStoWarps = 4;
constexpr int kStoTopCache = 2048;   // top-k lists up to this long are searched in shared memory

struct StochasticArgs {
  KvView kv;
  QView qv;
  const int32_t* top;     // [T][Hq][k_max] ascending, -1 padded
  int32_t k_max;
  const uint32_t* u;      // [T][Hq][m] random words
  int32_t m;
  int32_t* out_idx;       // [T][Hq][k_max + m]
  float* out_logw;        // [T][Hq][k_max + m]
  uint32_t* status;       // nullable
};

// Number of entries of the ascending list a[0..n) that are < x (a in shared or global memory).
__device__ __forceinline__ int count_below(const int32_t* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

struct StoSmem {
  uint32_t kept[kStoWarps][kStoMaxM];
  int32_t toks[kStoWarps][kStoMaxM];
  int32_t top[kStoWarps][kStoTopCache];
};

__global__ void __launch_bounds__(32 * kStoWarps) stochastic_select_kernel(StochasticArgs a) {
  extern __shared__ __align__(16) unsigned char sto_smem[];
  StoSmem& SM = *reinterpret_cast<StoSmem*>(sto_smem);
  auto& kept = SM.kept;
  auto& toks = SM.toks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t list = (int64_t)blockIdx.x * kStoWarps + warp;
  const int64_t nlists = (int64_t)a.qv.num_tokens * a.qv.hq;
  if (list >= nlists) return;
  const int t = (int)(list / a.qv.hq);
  // visible length of token t (sequence by binary search over q_indptr)
  int b = t;
  if (a.qv.q_indptr != nullptr) {
    int lo = 0, hi = a.kv.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.qv.q_indptr + mid) <= t) lo = mid; else hi = mid;
    }
    b = lo;
  }
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, false);
  const int L = (t >= si.t0 && t < si.t0 + si.n) ? kv_len_of(a.qv, si, t - si.t0) : 0;
  const int32_t* top = a.top + list * a.k_max;
  // the top list, searched many times below, is read once into shared memory when it fits;
  // its valid prefix (entries >= 0, ascending, < L) is then checked there
  const int32_t* topc = top;
  if (a.k_max <= kStoTopCache) {
#pragma unroll 4
    for (int i = lane; i < a.k_max; i += 32) SM.top[warp][i] = __ldg(top + i);
    __syncwarp();
    topc = SM.top[warp];
  }
  int ntop = 0;
  bool bad = false;
  for (int i = lane; i < a.k_max; i += 32) {
    const int32_t v = topc[i];
    if (v >= 0) {
      ntop = i + 1;
      bad |= v >= L || (i > 0 && topc[i - 1] >= v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ntop = max(ntop, __shfl_xor_sync(0xFFFFFFFFu, ntop, o));
  if (__any_sync(0xFFFFFFFFu, bad)) {   // not an ascending list of visible tokens: flag, keep nothing
    if (lane == 0 && a.status != nullptr) flag_status(a.status, TSD_DEV_BAD_INDEX);
    ntop = 0;
  }
  const int n = max(0, L - ntop);              // |R|
  const int m = min(a.m, n);
  const uint32_t* u = a.u + list * a.m;
  uint32_t* kr = kept[warp];
  // the random words go to shared memory first (the token array is free until the mapping),
  // so that Floyd's sequential steps do not wait on global loads
  uint32_t* us = reinterpret_cast<uint32_t*>(toks[warp]);
  for (int s = lane; s < m; s += 32) us[s] = __ldg(u + s);
  __syncwarp();
  // ---- Floyd: step s (j_s = n - m + s) keeps t_s = u_s mod (j_s + 1), or j_s if t_s was
  // kept before ----
  // All draws t_s are computed in parallel.  Then, repeatedly: steps before `from` are final;
  // the first step s >= from whose current value repeats an earlier kept value is a collision
  // of the sequential algorithm (the steps between keep their draws), so it keeps j_s, which
  // exceeds every earlier kept value and so never collides itself; the search resumes at s + 1.
  // With m << n collisions are rare and this is one or two parallel passes; after four passes
  // the remaining steps run in order (a warp scan per membership test), which bounds the cost
  // when m is not small against n.
  for (int s = lane; s < m; s += 32) kr[s] = us[s] % ((uint32_t)(n - m + s) + 1u);
  __syncwarp();
  for (int from = 0, passes = 0;; ++passes) {
    if (passes == 4) {   // many collisions (m not << n): the remaining steps in order
      for (int s = from; s < m; ++s) {
        const uint32_t v = kr[s];   // still the draw t_s: only steps before `from` were changed
        bool seen = false;
        for (int i = lane; i < s; i += 32) seen |= kr[i] == v;
        seen = __any_sync(0xFFFFFFFFu, seen);
        __syncwarp();
        if (seen && lane == 0) kr[s] = (uint32_t)(n - m + s);
        __syncwarp();
      }
      break;
    }
    int first = m;   // the first step >= from whose value repeats an earlier one (branch-free scans)
    for (int s = lane; s < m; s += 32) {
      const uint32_t v = kr[s];
      bool rep = false;
      for (int i = 0; i < s; ++i) rep |= kr[i] == v;
      if (rep && s >= from && s < first) first = s;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xFFFFFFFFu, first, o));
    if (first == m) break;
    __syncwarp();
    if (lane == 0) kr[first] = (uint32_t)(n - m + first);
    __syncwarp();
    from = first + 1;
  }
  // ---- sort the kept ranks (distinct) by counting, and map each to its token of R ----
  int32_t* tk = toks[warp];
  for (int i = lane; i < m; i += 32) {
    const uint32_t r = kr[i];
    int pos = 0;
    for (int j = 0; j < m; ++j) pos += kr[j] < r;
    // token = r + jstar, jstar = first index with top[j] - j > r (top ascending and distinct)
    int lo = 0, hi = ntop;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (topc[mid] - mid > (int)r) hi = mid; else lo = mid + 1;
    }
    tk[pos] = (int32_t)r + lo;
  }
  __syncwarp();
  // ---- merge S and the sample into one ascending list with log-weights ----
  const int width = a.k_max + a.m;
  int32_t* oi = a.out_idx + list * width;
  float* ow = a.out_logw + list * width;
  const float lw = m > 0 ? logf((float)n / (float)m) : 0.f;
  // top entries: lane l walks its contiguous chunk, one binary search for the chunk start
  // then a forward scan of the (ascending) samples
  {
    const int chunk = (ntop + 31) >> 5;
    const int i0 = lane * chunk, i1 = min(ntop, i0 + chunk);
    int pos = 0;   // sampled tokens below the current top entry
    if (i0 < i1) {
      const int32_t v0 = topc[i0];
      int lo = 0, hi = m;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (tk[mid] < v0) lo = mid + 1; else hi = mid;
      }
      pos = lo;
    }
    for (int i = i0; i < i1; ++i) {
      const int32_t v = topc[i];
      while (pos < m && tk[pos] < v) ++pos;
      oi[i + pos] = v;
      ow[i + pos] = 0.f;
    }
  }
  for (int i = lane; i < m; i += 32) {
    const int32_t v = tk[i];
    const int below = count_below(topc, ntop, v);
    oi[i + below] = v;
    ow[i + below] = lw;
  }
  for (int i = ntop + m + lane; i < width; i += 32) {
    oi[i] = -1;
    ow[i] = 0.f;
  }
}

cudaError_t launch_stochastic_select(const KvView& kv, const QView& qv, const int32_t* top, int k_max,
                                     const uint32_t* u, int m, int32_t* out_idx, float* out_logw, uint32_t* status,
                                     cudaStream_t stream) {
  StochasticArgs a;
  a.kv = kv;
  a.qv = qv;
  a.top = top;
  a.k_max = k_max;
  a.u = u;
  a.m = m;
  a.out_idx = out_idx;
  a.out_logw = out_logw;
  a.status = status;
  const int64_t nlists = (int64_t)qv.num_tokens * qv.hq;
  const int64_t grid = (nlists + kStoWarps - 1) / kStoWarps;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(stochastic_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(StoSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  stochastic_select_kernel<<<(unsigned)grid, 32 * kStoWarps, sizeof(StoSmem), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tsd
