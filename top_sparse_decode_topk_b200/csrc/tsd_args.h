// Kernel argument blocks of libtsd (passed by value to the kernels).
#pragma once

#include <stdint.h>

#include "tsd_common.cuh"

namespace tsd {

struct DecodeArgs {
  KvView kv;
  QView qv;
  const int32_t* idx;   // sparse: [T][Hq][k_max]; dense: unused
  const float* logw;    // sparse, optional: [T][Hq][k_max] natural-log weight of each entry
  int32_t k_max;
  int32_t span;         // sparse: entries per list per split (E); dense: tokens per window (W)
  int32_t nsplit;
  int32_t lists_per_cta;
  int32_t list_groups;
  void* out;
  int32_t out_f32;
  float* lse;
  uint32_t* status;
  uint32_t* counters;
  float2* part_ml;
  float* part_acc;
  uint32_t* sched;      // sparse, persistent kernel: [0] next task to hand out, [1] warps done (zero region)
  int32_t persistent;   // sparse: 1 runs the persistent kernel (span = E, a multiple of 32)
};

struct TopkArgs {
  KvView kv;
  QView qv;
  int32_t k_max;
  const int32_t* k_per_token;
  int32_t* out_idx;
  int32_t* out_count;
  float* out_scores;    // optional [T][Hq][k_max]: the kept tokens' scores (-inf in the padding)
  float* scores;
  int64_t score_stride;
  float* samples;         // [T][Hq][sample_stride]: score of every 2^sample_shift-th token
  int64_t sample_stride;
  int32_t sample_shift;
  int32_t filter;         // 1: the sample pre-pass, thresholds and candidate appends run (exact indexer)
  uint32_t* lo_key;       // [T][Hq] candidate threshold keys (filter)
  uint2* cand;            // [T][Hq][kTopkCandCap] (key, index) candidates (filter)
  uint32_t* cand_cnt;     // [T][Hq] candidate slots reserved (zero region; the selection clears it)
  int2* meta;             // [T][Hq] (kv_len, k) of each list (filter: pre-pass -> selection)
  int32_t prepass_splits; // filter: CTAs sharing one (sequence, kv head, list group)'s sample tiles
  int32_t* queue;         // filter: [T][Hq] lists the candidate kernel left to the row paths
  uint32_t* queue_cnt;    // filter: their number (zero region; the last queue CTA clears it)
  uint32_t* queue_done;   // filter: queue CTAs finished (zero region; cleared with queue_cnt)
  int32_t queue_ctas;     // filter: CTAs of the queue pass
  const uint16_t* label;    // label indexer: [rows][label_r] bf16 label cache (NULL: the exact indexer)
  const int32_t* channels;  // label indexer: [Hkv][label_r] channel ids
  int32_t label_r;          // label indexer: channels per kv head
  int32_t lists_per_cta;
  int32_t list_groups;
  int32_t window;
  uint32_t* status;
};

}  // namespace tsd
