// Work decomposition and workspace layout of libtsd (host and device).
//
// Workspace layout (bytes from the start; every region 256-byte aligned):
//   [0, 256)              header: device status word (uint32) at offset 0; the persistent
//                         sparse kernel's task and done counters (uint32) at offsets 4 and 8;
//                         the filtered indexer's queue count and queue-CTA counter (uint32) at
//                         offsets 16 and 20; the rest reserved
//   counters              uint32, one per list (token x q head): arrival counters of the
//                         split-K merge, or the filtered indexer's candidate counters (and the
//                         pre-pass's arrival counters); zero between calls
//   -- everything above is the "zero region": it must be zero when a call starts and every
//      call leaves it zero --
//   decode partials       float2 [T][Hq][nsplit] (running max, running sum; base-2 units)
//                         float  [T][Hq][nsplit][128] (unnormalised output rows)
//   top-k scores          float  [T][Hq][score_stride] (fp32 q.K of every visible token)
//   top-k score samples   float  [T][Hq][sample_stride]: every 2^sample_shift-th token's score
//                         (its strided sample for the selection's threshold)
//   filtered indexer      thresholds, candidates, (kv_len, k) and the queue (TopkLayout)
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "tsd.h"

#define TSD_DEV_BAD_SEQ_BIT TSD_DEV_BAD_SEQ

namespace tsd {

constexpr int kMaxSplits = 256;         // split-K partials per (token, head)
constexpr int kMaxEntriesPerSplit = 1024;  // bound used for the largest supported k

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Shapes {
  int64_t batch, hkv, hq, group, tokens, max_tokens, max_seq_len;
};

// Room for one arrival counter per list (token x q head), which also covers one per
// (sequence, kv head, list group).
inline size_t zero_region_bytes(const Shapes& s) {
  const int64_t toks = s.batch * s.max_tokens > s.tokens ? s.batch * s.max_tokens : s.tokens;
  return 256 + align256((size_t)toks * s.hq * sizeof(uint32_t));
}

// Longest index list tsd_sparse_decode accepts (kMaxSplits chunks of at most
// kMaxEntriesPerSplit entries).
constexpr int kMaxSparseK = kMaxSplits * kMaxEntriesPerSplit;

// Sparse decode: every list (token x q head) is cut into C tasks of E entries (E a
// multiple of 16, the row tile); a task is one warp and a CTA runs kSpTasksPerCta tasks.
// Every task takes about the same time, so a grid that spills a little into a second wave
// of resident CTAs costs nearly a whole extra wave.  The plan therefore takes the smallest
// E whose tasks fit one wave (kSpCtasPerSm CTAs on each SM).  When even one task per list
// leaves that wave well under-filled (many lists, as with several decode tokens per
// sequence), it cuts the lists finer instead, about two tasks per resident warp, and lets
// the lists of unequal length even out.  C stays <= kMaxSplits either way.
struct SparsePlan {
  int lists;     // list slots per (sequence, kv head): G x max tokens per sequence
  int entries;   // E
  int nsplit;    // C
  int stream;    // 1: the persistent kernel (tasks handed out through a counter), 0: one task per warp
};

constexpr int kSpTasksPerCta = 4;   // warps per sparse-decode CTA, one task each
constexpr int kSpStages = 3;        // 16-row tiles in each warp's shared-memory ring (8 KB each)
constexpr int kSpCtasPerSm = 2;     // resident sparse-decode CTAs per SM (its launch bounds)

inline SparsePlan plan_sparse(const Shapes& s, int k_max, int num_sms) {
  SparsePlan p;
  p.lists = (int)(s.group * s.max_tokens);
  const int64_t slots = (int64_t)num_sms * kSpCtasPerSm;
  const int64_t units = s.batch * s.hkv * p.lists;
  const int kr = (k_max + 15) / 16 * 16;
  constexpr int NW = kSpTasksPerCta;
  int e = 16;
  for (; e < kr; e += 16) {
    const int64_t ns = (k_max + e - 1) / e;
    if (ns <= kMaxSplits && (units * ns + NW - 1) / NW <= slots) break;
  }
  const int64_t ctas = (units * ((k_max + e - 1) / e) + NW - 1) / NW;
  if (4 * ctas < 3 * slots) {   // one wave would be under-filled: about two tasks per warp
    const double total = (double)s.tokens * s.hq * k_max;
    e = (int)(total / (2.0 * NW * (double)slots));
    e = (e + 15) / 16 * 16;
    if (e < 16) e = 16;
    if (e > kMaxEntriesPerSplit) e = kMaxEntriesPerSplit;
    if (e > kr) e = kr;
    if ((k_max + e - 1) / e > kMaxSplits) e = ((k_max + kMaxSplits - 1) / kMaxSplits + 15) / 16 * 16;
  }
  p.entries = e;
  p.nsplit = (k_max + e - 1) / e;
  p.stream = 0;
  return p;
}

// Persistent sparse decode: kSsCtasPerSm CTAs of kSsWarpsPerCta warps on every SM, each warp
// taking (list, chunk) tasks from a counter until none is left, with the next task's first
// windows prefetched while the current one drains.  Lists are cut into chunks of E entries (a
// multiple of the 32-entry window): E is sized for about six tasks per warp, so that the warps
// finish together, within [64, 512] so that a task is long enough to hide its start and the
// split-K partials stay a few percent of the traffic.
constexpr int kSsWarpsPerCta = 4;
constexpr int kSsCtasPerSm = 2;

inline SparsePlan plan_sparse_stream(const Shapes& s, int k_max, int num_sms, int entries_override) {
  SparsePlan p;
  p.lists = (int)(s.group * s.max_tokens);
  const double warps = (double)num_sms * kSsCtasPerSm * kSsWarpsPerCta;
  const double work = (double)s.tokens * s.hq * k_max;
  const int kr = (k_max + 31) / 32 * 32;
  int e = entries_override > 0 ? entries_override : (int)(work / (warps * 6.0));
  e = (e + 31) / 32 * 32;
  if (entries_override <= 0) {
    if (e < 64) e = 64;
    if (e > 512) e = 512;
  }
  if (e < 32) e = 32;
  if (e > kr) e = kr;
  if ((k_max + e - 1) / e > kMaxSplits) e = ((k_max + kMaxSplits - 1) / kMaxSplits + 31) / 32 * 32;
  p.entries = e;
  p.nsplit = (k_max + e - 1) / e;
  p.stream = 1;
  return p;
}

// Dense decode and top-k scoring: up to 16 lists per CTA (the mma M dimension) and a window
// of W tokens (a multiple of the 64-token tile) per (sequence, kv head, list group).  `wave`
// is the number of resident CTAs (CTAs per SM x SMs).
struct DensePlan {
  int lists_per_cta;
  int list_groups;
  int window;
  int nsplit;
};

constexpr int kDenseMaxLists = 16;
constexpr int kDnCtasPerSm = 3;    // resident dense-decode CTAs per SM (its launch bounds)
constexpr int kScCtasPerSm = 6;    // resident top-k scoring CTAs per SM, warp-MMA kernel (its launch bounds;
                                   // bf16 queries: fp32 queries' second query tile leaves room for 5)
constexpr int kScTcCtasPerSm = 6;  // the same for the tcgen05 scoring kernel
constexpr int kScoreCtasPerSm = kScCtasPerSm;
static_assert(kScTcCtasPerSm == kScCtasPerSm, "both scoring kernels share one window plan");
// Tokens per CTA at most.  Windows are sized on max_seq_len, so on a ragged batch (lengths
// 8K-128K against a 128K bound) about half the windows lie past their sequence's end and exit at
// once, and the live ones run in coarse waves.  Measured on the ragged batch (CUDA graphs, L2
// flushed): the top-k leg took 1677 us with 8192-token windows and 1585 us with 4096 (2048: 1589);
// dense decode took 2006 us with 8192 and 1979 us with 4096, but on the Qwen2.5-72B shape 4096
// forced a third wave of dense CTAs (392 -> 405 us).  So the scoring kernels cap at 4096 tokens and
// dense decode at 8192.
constexpr int64_t kMaxWindowDense = 8192;
constexpr int64_t kMaxWindowScore = 4096;

// Window of `ns` windows over max_seq_len, rounded up to whole 64-token tiles.
inline int64_t dense_window(int64_t max_seq_len, int64_t ns) {
  const int64_t w = (max_seq_len + ns - 1) / ns;
  return (w + 63) / 64 * 64;
}

inline DensePlan plan_dense(const Shapes& s, int64_t wave, int64_t kMaxWindow = kMaxWindowDense) {
  DensePlan p;
  const int64_t m = s.group * s.max_tokens;
  p.lists_per_cta = (int)(m < kDenseMaxLists ? m : kDenseMaxLists);
  p.list_groups = (int)((m + p.lists_per_cta - 1) / p.lists_per_cta);
  const int64_t units = s.batch * s.hkv * p.list_groups;
  int64_t max_ns = (s.max_seq_len + 63) / 64;
  if (max_ns > kMaxSplits) max_ns = kMaxSplits;
  if (max_ns < 1) max_ns = 1;
  // Every CTA streams about the same number of tiles: size the grid to two whole waves of
  // `wave` resident CTAs.
  int64_t ns = 2 * wave / units;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  if (dense_window(s.max_seq_len, ns) > kMaxWindow) {
    // Few units over a long max_seq_len (a large or ragged batch).  Windows are sized on
    // max_seq_len while sequences may be much shorter (windows past a sequence's end exit at
    // once), and a long sequence cut into few windows leaves its CTAs running alone at the
    // end: cap the window at kMaxWindow and, above that floor, take the split count whose
    // whole waves x (window + one tile of merge and prologue) is least.
    int64_t lo = (s.max_seq_len + kMaxWindow - 1) / kMaxWindow;
    if (lo > max_ns) lo = max_ns;
    int64_t hi = 4 * wave / units + 1;
    if (hi > max_ns) hi = max_ns;
    if (hi < lo) hi = lo;
    int64_t best = -1;
    for (int64_t n = lo; n <= hi; ++n) {
      const int64_t w = dense_window(s.max_seq_len, n);
      const int64_t nse = (s.max_seq_len + w - 1) / w;
      const int64_t cost = ((units * nse + wave - 1) / wave) * (w + 64);
      if (best < 0 || cost < best) { best = cost; ns = n; }
    }
  }
  const int64_t w = dense_window(s.max_seq_len, ns);
  p.window = (int)w;
  p.nsplit = (int)((s.max_seq_len + w - 1) / w);
  return p;
}

struct DecodeLayout {
  size_t off_counters, off_ml, off_acc, total;
};

inline DecodeLayout decode_layout(const Shapes& s, int nsplit) {
  DecodeLayout l;
  l.off_counters = 256;
  size_t off = zero_region_bytes(s);
  l.off_ml = off;
  off += align256((size_t)s.tokens * s.hq * nsplit * 2 * sizeof(float));
  l.off_acc = off;
  off += align256((size_t)s.tokens * s.hq * nsplit * 128 * sizeof(float));
  l.total = off;
  return l;
}

// The scoring kernels also write every 2^sample_shift-th token's score into a compact sample
// row, so that the selection reads its sample contiguously.  The stride is 32 tokens, doubled
// while the sample would exceed kMaxSample scores.
constexpr int64_t kMaxSample = 4096;

// Candidates of the exact indexer (tsd_topk_select): the scoring kernel also appends every
// (key, index) at or above a list's sampled threshold, at most kTopkCandCap per list.
constexpr int kTopkCandCap = 8192;

struct TopkLayout {
  size_t off_scores;
  int64_t score_stride;
  size_t off_samples;
  int32_t sample_shift;
  int64_t sample_stride;
  size_t off_lo;      // uint32 [T][Hq]: each list's candidate threshold key
  size_t off_cand;    // uint2 [T][Hq][kTopkCandCap]: (key, index) candidates
  size_t off_meta;    // int2 [T][Hq]: each list's (kv_len, k), written by the pre-pass
  size_t off_queue;   // int32 [T][Hq]: lists the candidate kernel leaves to the row paths
  size_t total;
};

inline TopkLayout topk_layout(const Shapes& s) {
  TopkLayout l;
  l.score_stride = (s.max_seq_len + 3) / 4 * 4;
  l.off_scores = zero_region_bytes(s);
  l.sample_shift = 5;
  while (((s.max_seq_len + (1LL << l.sample_shift) - 1) >> l.sample_shift) > kMaxSample) ++l.sample_shift;
  l.sample_stride = (((s.max_seq_len + (1LL << l.sample_shift) - 1) >> l.sample_shift) + 3) / 4 * 4;
  l.off_samples = l.off_scores + align256((size_t)s.tokens * s.hq * l.score_stride * sizeof(float));
  l.off_lo = l.off_samples + align256((size_t)s.tokens * s.hq * l.sample_stride * sizeof(float));
  l.off_cand = l.off_lo + align256((size_t)s.tokens * s.hq * sizeof(uint32_t));
  l.off_meta = l.off_cand + align256((size_t)s.tokens * s.hq * kTopkCandCap * 2 * sizeof(uint32_t));
  l.off_queue = l.off_meta + align256((size_t)s.tokens * s.hq * 2 * sizeof(int32_t));
  l.total = l.off_queue + align256((size_t)s.tokens * s.hq * sizeof(int32_t));
  return l;
}

}  // namespace tsd
