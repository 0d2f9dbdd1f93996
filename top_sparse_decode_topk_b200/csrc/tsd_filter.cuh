// Device helpers of the candidate filter shared by the exact indexer (tsd_topk.cu) and the
// label indexer (tsd_label.cu): per-list thresholds from a strided sample, a list's kept count,
// and the warp-collective candidate append.
#pragma once

#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"
#include "tsd_plan.h"

namespace tsd {

constexpr int kThrMaxSamples = 2048;   // 64 per lane

// Longest list the candidate selection covers (its bitmaps of the list's tokens): calls whose
// max_seq_len is longer take the unfiltered form.
constexpr int kTopkCandMaxLen = 131072;

// Threshold key of one list from its ns sample scores (one warp): bit by bit from the top, the
// r-th largest sample key with its low 16 bits cleared, r the expected count above the k-th
// score plus 4 standard deviations plus 4 -- with overwhelming probability at least k of the
// list's scores reach it.  Lists of at most kTopkCandCap / 2 tokens take every score (lo = 0); a
// list the filter cannot serve (k = 0, k = L, too many expected candidates, or more samples than
// the warp holds) gets lo = 0xFFFFFFFF, which only the largest NaN key reaches, and the
// selection takes its other paths.
__device__ inline uint32_t list_threshold(const float* samp, int L, int k, int shift, bool enabled, int lane) {
  constexpr unsigned FULL = 0xFFFFFFFFu;
  if (!(k > 0 && k < L && enabled)) return 0xFFFFFFFFu;
  if (L <= kTopkCandCap / 2) return 0u;   // leaves room for the pools' holes
  const int ns = (L + (1 << shift) - 1) >> shift;
  const float mean = (float)ns * (float)k / (float)L;
  const int r = (int)ceilf(mean + 4.f * sqrtf(mean) + 4.f);
  if (!(ns <= kThrMaxSamples && r < ns && (int64_t)r * L <= (int64_t)kTopkCandCap * ns * 3 / 4)) return 0xFFFFFFFFu;
  uint32_t key[kThrMaxSamples / 32];
#pragma unroll
  for (int i = 0; i < kThrMaxSamples / 32; ++i) {
    const int j = 32 * i + lane;
    key[i] = j < ns ? score_key(__ldcg(samp + j)) : 0u;
  }
  // 16 bits (sign, exponent, 7 mantissa bits): the threshold then sits at most 2^-7 of its
  // value below the sample's r-th largest, which adds few candidates; eight partial counts keep
  // the chains of dependent adds short
  uint32_t prefix = 0u;
  for (int bit = 31; bit >= 16; --bit) {
    const uint32_t trial = prefix | (1u << bit);
    int c8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kThrMaxSamples / 32; ++i) c8[i & 7] += key[i] >= trial;
    int c = ((c8[0] + c8[1]) + (c8[2] + c8[3])) + ((c8[4] + c8[5]) + (c8[6] + c8[7]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(FULL, c, o);
    if (c >= r) prefix = trial;
  }
  return prefix;
}

// kept count k = min(k_t, L) of query token t with visible length L
__device__ __forceinline__ int list_k(const TopkArgs& a, int t, int L) {
  int kreq = a.k_max;
  if (a.k_per_token != nullptr) {
    kreq = __ldg(a.k_per_token + t);
    kreq = kreq < 0 ? 0 : (kreq > a.k_max ? a.k_max : kreq);
  }
  return kreq < L ? kreq : L;
}

// Warp-collective: every lane calls it with the same pool [pn, pe) of reserved slots.  Lanes with
// `cand` append (key(sc), tok) to the list's buffer in lane order; when the pool runs short, lane
// 0 reserves whole chunks of `chunk` slots with one atomic on the list's counter.
__device__ __forceinline__ void warp_append(bool cand, float sc, uint32_t tok, uint32_t& pn, uint32_t& pe,
                                            uint32_t* cnt, uint2* buf, int lane, uint32_t chunk) {
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
  if (bal == 0u) return;
  const uint32_t n = __popc(bal);
  const uint32_t room = pe - pn;
  uint32_t fresh = 0u, want = 0u;
  if (n > room) {
    want = (n - room + chunk - 1) / chunk * chunk;
    if (lane == 0) fresh = atomicAdd(cnt, want);
    fresh = __shfl_sync(0xFFFFFFFFu, fresh, 0);
  }
  if (cand) {
    const uint32_t i = __popc(bal & ((1u << lane) - 1u));
    const uint32_t slot = i < room ? pn + i : fresh + (i - room);
    if (slot < (uint32_t)kTopkCandCap) buf[slot] = make_uint2(score_key(sc), tok);
  }
  if (n > room) {
    pn = fresh + (n - room);
    pe = fresh + want;
  } else {
    pn += n;
  }
}

}  // namespace tsd
