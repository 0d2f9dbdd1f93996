// Work decomposition and workspace layout of libtsd (host and device).
//
// Workspace layout (bytes from the start; every region 256-byte aligned):
//   [0, 256)              header: device status word (uint32) at offset 0; sparse-decode
//                         work-unit counter at byte 4 and finished-CTA counter at byte 8
//   counters              uint32 [batch][num_kv_heads][group * max_tokens]: arrival counters
//                         of the split-K merge, one per list group (zero between calls)
//   -- everything above is the "zero region": it must be zero when a call starts and every
//      call leaves it zero --
//   decode partials       float2 [T][Hq][nsplit] (running max, running sum; base-2 units)
//                         float  [T][Hq][nsplit][128] (unnormalised output rows)
//   top-k scores          float  [T][Hq][score_stride] (fp32 q.K of every visible token)
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "tsd.h"

#define TSD_DEV_BAD_SEQ_BIT TSD_DEV_BAD_SEQ

namespace tsd {

constexpr int kMaxListsPerCta = 32;     // query lists (token x q head) handled by one CTA
constexpr int kSparseMaxLists = 16;     // sparse decode: lists per work unit (one half-warp each at least)
constexpr int kDecodeThreads = 256;     // 8 warps = 32 groups of 8 lanes
constexpr int kRowsPerTile = 16;        // K/V rows per pipeline stage
constexpr int kStages = 4;              // cp.async pipeline depth
constexpr int kMaxEntriesPerCta = 1024; // sparse: lists x entries per CTA
constexpr int kBitmapWords = 1024;      // sparse: dedupe bitmap spans 32768 tokens
constexpr int kMaxSplits = 256;         // split-K partials per (token, head)
constexpr int kSparseEntriesTarget = 256;  // sparse: entries (all lists) a CTA aims for
constexpr int kScoreThreads = 256;
constexpr int kSelectThreads = 512;
constexpr int kScoreTokensPerCta = 1024;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Shapes {
  int64_t batch, hkv, hq, group, tokens, max_tokens, max_seq_len;
};

inline int list_groups(const Shapes& s) {
  int64_t m = s.group * s.max_tokens;
  return (int)((m + kMaxListsPerCta - 1) / kMaxListsPerCta);
}

// Room for one counter per list, enough for any split of the lists into groups.
inline size_t zero_region_bytes(const Shapes& s) {
  return 256 + align256((size_t)s.batch * s.hkv * s.group * s.max_tokens * sizeof(uint32_t));
}

// Longest index list tsd_sparse_decode accepts (kMaxSplits chunks of at most
// kMaxEntriesPerCta entries).
constexpr int kMaxSparseK = kMaxSplits * kMaxEntriesPerCta;

// Sparse decode: entries per list per CTA (E) and number of splits.
struct SparsePlan {
  int lists_per_cta;
  int list_groups;
  int entries;   // E
  int nsplit;
};

inline SparsePlan plan_sparse(const Shapes& s, int k_max) {
  SparsePlan p;
  const int64_t m = s.group * s.max_tokens;
  int lists = (int)(m < kSparseMaxLists ? m : kSparseMaxLists);
  const int kr = (k_max + 15) / 16 * 16;
  int e = (kSparseEntriesTarget / lists + 15) / 16 * 16;
  if (e < 16) e = 16;
  if (e > kr) e = kr;
  int ns = (k_max + e - 1) / e;
  if (ns > kMaxSplits) {
    e = ((k_max + kMaxSplits - 1) / kMaxSplits + 15) / 16 * 16;   // long lists: bigger chunks
    ns = (k_max + e - 1) / e;
  }
  p.lists_per_cta = lists;
  p.list_groups = (int)((m + lists - 1) / lists);
  p.entries = e;
  p.nsplit = ns;
  return p;
}

// Dense decode: tokens per CTA window and number of windows.
struct DensePlan {
  int lists_per_cta;
  int list_groups;
  int window;
  int nsplit;
};

inline DensePlan plan_dense(const Shapes& s) {
  DensePlan p;
  int64_t m = s.group * s.max_tokens;
  p.lists_per_cta = (int)(m < kMaxListsPerCta ? m : kMaxListsPerCta);
  p.list_groups = list_groups(s);
  int w = 1024;
  int ns = (int)((s.max_seq_len + w - 1) / w);
  while (ns > kMaxSplits) {
    w *= 2;
    ns = (int)((s.max_seq_len + w - 1) / w);
  }
  p.window = w;
  p.nsplit = ns;
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

struct TopkLayout {
  size_t off_scores;
  int64_t score_stride;
  size_t total;
};

inline TopkLayout topk_layout(const Shapes& s) {
  TopkLayout l;
  l.score_stride = (s.max_seq_len + 3) / 4 * 4;
  l.off_scores = zero_region_bytes(s);
  l.total = l.off_scores + align256((size_t)s.tokens * s.hq * l.score_stride * sizeof(float));
  return l;
}

}  // namespace tsd
