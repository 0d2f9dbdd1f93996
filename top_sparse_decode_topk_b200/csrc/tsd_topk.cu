// Exact top-k token selection ("Oracle Top-K") for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?",
// gist.science summary, section 2): for every query token t and q head h keep
// the k tokens with the largest q.K, exactly; ties go to the lower token index
// and the kept indices are written in ascending order.
//
// Two kernels:
//  * topk_score_kernel -- one CTA per (sequence, kv head, list group of <= 16 lists, window of
//    tokens).  A producer warp streams 64-token K tiles into shared memory with TMA; four
//    consumer warps score them against the lists' queries on the tensor cores (mma.sync,
//    bf16 in, fp32 accumulate) and write fp32 scores.  Each K row is read from HBM once for
//    every query of the GQA group and every decode token of the sequence.
//  * topk_select_kernel -- one CTA per (t, h).  Scores map to order-preserving
//    uint32 keys; an 11-bit histogram finds the bin holding the k-th key,
//    further digit passes narrow it until the candidates fit shared memory, a
//    radix select over the candidates gives the exact k-th key T, and a final
//    ordered pass keeps every key > T plus the lowest-index keys == T, writing
//    them in ascending token order with block-wide prefix sums.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "tsd_args.h"
#include "tsd_common.cuh"
#include "tsd_kvtile.cuh"
#include "tsd_umma.cuh"

namespace tsd {

constexpr int kSelectThreads = 512;   // one CTA per (token, head)
constexpr int kSelBins = 2048;
constexpr int kCandMax = 16384;
constexpr int kSelPerThread = 16;                 // scores per thread per tile (4 x float4)


// ---------------------------------------------------------------------------
// Scoring on tensor cores
// ---------------------------------------------------------------------------
// One CTA per (sequence b, kv head g, list group lg, window of W tokens).  A producer warp
// streams 64-token K tiles through a 2-stage ring (TMA, tsd_kvtile.cuh); each of the 4
// consumer warps scores 16 tokens of every tile against the CTA's 16 query rows with
// mma.m16n8k16 (bf16 inputs, fp32 accumulation; fp32 queries as bf16 hi + lo) and writes
// the unscaled fp32 dots of tokens below each list's kv_len.  The streaming rate grows with
// resident CTAs rather than ring depth, so the ring is short and 5 CTAs share an SM (the
// fp32 remainder tile is only allocated for fp32 queries).
constexpr int kScConsumers = 4;
constexpr int kScThreads = 32 * (kScConsumers + 1);

// shared-memory layout (offsets from a 1024-aligned base): stages, q hi, [q lo], barriers
template <bool QF32, int NST>
struct ScLayout {
  static constexpr int kStages = NST;
  static constexpr size_t qhi = (size_t)NST * kTileBytesKV;
  static constexpr size_t qlo = qhi + kQTileBytes;
  static constexpr size_t bars = qhi + (QF32 ? 2 : 1) * kQTileBytes;
  static constexpr size_t bytes = bars + 2 * NST * sizeof(uint64_t) + 16;
};
constexpr int kScStages = 2;
static_assert(ScLayout<true, kScStages>::bytes + 1024 <= 228 * 1024 / kScCtasPerSm, "scoring CTAs per SM");

template <bool QF32>
__global__ void __launch_bounds__(kScThreads, kScCtasPerSm) topk_score_kernel(TopkArgs a, const __grid_constant__ KvMaps maps) {
  using Lay = ScLayout<QF32, kScStages>;
  extern __shared__ __align__(1024) unsigned char smem_sc[];
  unsigned char* stages = smem_sc;
  unsigned char* qhi = smem_sc + Lay::qhi;
  unsigned char* qlo = smem_sc + Lay::qlo;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_sc + Lay::bars);
  uint64_t* empty = full + kScStages;
  uint32_t* abort_flag = reinterpret_cast<uint32_t*>(empty + kScStages);
  const int win = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, win == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;
  const int tok0 = win * a.window;
  const int tok_end = min(tok0 + a.window, si.len);
  if (tok_end <= tok0) return;
  const int ntiles = (tok_end - tok0 + kTileTok - 1) / kTileTok;
  const bool use_tma = a.kv.page_table == nullptr || a.kv.page_shift >= 3;
  if (smem_u32(stages) & 1023u) {
    if (threadIdx.x == 0) flag_status(a.status, TSD_DEV_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScStages; ++s) {
      mbar_init(&full[s], use_tma ? 1 : 32);
      mbar_init(&empty[s], kScConsumers);
    }
    mbar_fence_init();
    *abort_flag = 0;
  }
  store_q_tile(a.qv, si, g, G, lg * a.lists_per_cta, nlists, qhi, QF32 ? qlo : nullptr, threadIdx.x, kScThreads);
  __syncthreads();

  if (warp == kScConsumers) {
    produce_tiles<kScStages, kTileBytesKV, false>(a.kv, maps, b, g, tok0, tok_end, ntiles, stages, full,
                                                  empty, abort_flag, use_tma, lane, a.status);
    return;
  }
  // this lane's query rows m = lane/4 and lane/4 + 8: visible length and score row
  int kvl[2];
  float* srow[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int m = (lane >> 2) + 8 * hr;
    kvl[hr] = 0;
    srow[hr] = a.scores;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int j = mg / G;
      kvl[hr] = min(kv_len_of(a.qv, si, j), tok_end);
      srow[hr] = a.scores + ((int64_t)(si.t0 + j) * a.qv.hq + g * G + (mg - j * G)) * a.score_stride;
    }
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    if (!consume_wait<kScStages>(full, abort_flag, tile, lane, a.status)) break;
    float sc[2][4];
    qk_tile<QF32>(qhi, qlo, stages + (size_t)(tile % kScStages) * kTileBytesKV, warp, lane, sc);
    const int tbase = tok0 + tile * kTileTok + 16 * warp + 2 * (lane & 3);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int tk = tbase + 8 * nt;   // even: the pair (tk, tk + 1) is 8-byte aligned
        if (tk + 1 < kvl[hr]) {
          *reinterpret_cast<float2*>(srow[hr] + tk) = make_float2(sc[nt][2 * hr], sc[nt][2 * hr + 1]);
        } else if (tk < kvl[hr]) {
          srow[hr][tk] = sc[nt][2 * hr];
        }
      }
    // the stores consume every fragment read from the stage: release it to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[tile % kScStages]);
  }
}

// ---------------------------------------------------------------------------
// Scoring on the fifth-generation tensor cores (tcgen05)
// ---------------------------------------------------------------------------
// The same work as topk_score_kernel with the MMA transposed: D[64 tokens x 16 lists] =
// K_tile[64 x 128] x Q[16 x 128]^T, one tcgen05.mma (M = 64, N = 16, K = 16) per k-step,
// issued by a single thread with both operands read from shared memory -- the K tile exactly
// as the TMA load wrote it (K-major, 128-byte swizzle) and the query tile in the same
// layout -- and the fp32 accumulator in tensor memory.
//   warp 0     : TMA producer, 64-token K tiles into a 2-stage ring;
//   warp 1     : allocates 32 tensor-memory columns (two 16-column accumulators) and, from one
//                lane, issues the MMAs of each tile and commits them to the stage's "empty"
//                barrier and the accumulator's "full" barrier;
//   warps 2..5 : epilogue: with M = 64, rows 16 q .. 16 q + 15 of the accumulator sit in
//                tensor-memory lanes 32 q .. 32 q + 15, so the warp reading lane quarter q
//                gets 16 tokens x 16 lists with tcgen05.ld, releases the accumulator and stores
//                the lists' scores.
// Every wait is bounded; on a timeout the CTA flags TSD_DEV_TIMEOUT, drains the MMAs it issued
// and frees its tensor memory before returning.
// Measured against topk_score_kernel on llama3_8b (top-k leg, CUDA events): 155.6 vs 144.4 us
// at 5 CTAs per SM (M = 128 tiles at 3 CTAs per SM: 171.0 us).  The kernel is bound by the K
// stream, and the extra hop through the MMA issuer and tensor memory costs more than the
// warp-level MMAs it replaces, so it is selected only with TSD_SCORE_KERNEL=tcgen05.
constexpr int kTcTile = 64;                        // tokens per tile = the MMA's M (64 or 128)
constexpr int kTcStages = 2;
constexpr int kTcStageBytes = 2 * kTcTile * 128;   // two 128-byte halves of kTcTile rows
constexpr int kTcThreads = 192;
constexpr int kTcCtasPerSm = kScTcCtasPerSm;
// Accumulator rows per tensor-memory lane quarter: with M = 128 row r is lane r; with M = 64
// rows 16 q .. 16 q + 15 sit in lanes 32 q .. 32 q + 15 (the single-CTA M = 64 layout).
constexpr int kTcRowsPerQuarter = kTcTile / 4;
constexpr uint32_t kTcCols = 32;

template <bool QF32>
struct TcLayout {
  static constexpr size_t qhi = (size_t)kTcStages * kTcStageBytes;
  static constexpr size_t qlo = qhi + kQTileBytes;
  static constexpr size_t bars = qhi + (QF32 ? 2 : 1) * kQTileBytes;
  static constexpr size_t lists = bars + (2 * kTcStages + 4) * sizeof(uint64_t) + 16;   // score rows, lengths
  static constexpr size_t bytes = lists + 16 * sizeof(int64_t) + 16 * sizeof(int);
};
static_assert(TcLayout<true>::bytes + 1024 <= 228 * 1024 / kTcCtasPerSm, "tensor-core scoring CTAs per SM");

template <bool QF32>
__global__ void __launch_bounds__(kTcThreads, kTcCtasPerSm)
    topk_score_tc_kernel(TopkArgs a, const __grid_constant__ KvMaps maps) {
  using Lay = TcLayout<QF32>;
  extern __shared__ __align__(1024) unsigned char smem_tc[];
  unsigned char* stages = smem_tc;
  unsigned char* qhi = smem_tc + Lay::qhi;
  unsigned char* qlo = smem_tc + Lay::qlo;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_tc + Lay::bars);
  uint64_t* empty = full + kTcStages;
  uint64_t* accf = empty + kTcStages;
  uint64_t* acce = accf + 2;
  uint32_t* abort_flag = reinterpret_cast<uint32_t*>(acce + 2);
  uint32_t* tmem_slot = abort_flag + 1;
  int64_t* s_srow = reinterpret_cast<int64_t*>(smem_tc + Lay::lists);
  int* s_kvl = reinterpret_cast<int*>(s_srow + 16);
  const int win = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, win == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;
  const int tok0 = win * a.window;
  const int tok_end = min(tok0 + a.window, si.len);
  if (tok_end <= tok0) return;
  const int ntiles = (tok_end - tok0 + kTcTile - 1) / kTcTile;
  const bool use_tma = a.kv.page_table == nullptr || a.kv.page_shift >= 3;
  if (smem_u32(stages) & 1023u) {   // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) flag_status(a.status, TSD_DEV_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], use_tma ? 1 : 32);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&accf[s], 1);
      mbar_init(&acce[s], 4);
    }
    mbar_fence_init();
    *abort_flag = 0;
  }
  if (threadIdx.x < 16) {
    const int m = threadIdx.x;
    s_kvl[m] = 0;
    s_srow[m] = 0;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int j = mg / G;
      s_kvl[m] = min(kv_len_of(a.qv, si, j), tok_end);
      s_srow[m] = ((int64_t)(si.t0 + j) * a.qv.hq + g * G + (mg - j * G)) * a.score_stride;
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTcCols);
    tmem_relinquish();
  }
  store_q_tile(a.qv, si, g, G, lg * a.lists_per_cta, nlists, qhi, QF32 ? qlo : nullptr, threadIdx.x, kTcThreads);
  // the query tile is read by the tensor cores (async proxy): order the generic stores first
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    produce_tiles<kTcStages, kTcStageBytes, false, kTcTile>(a.kv, maps, b, g, tok0, tok_end, ntiles, stages, full,
                                                            empty, abort_flag, use_tma, lane, a.status);
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kTcTile, 16);
      const uint32_t qh = smem_u32(qhi), ql = smem_u32(qlo);
      int issued = 0;
      for (int tile = 0; tile < ntiles; ++tile) {
        const int s = tile % kTcStages, acc = tile & 1;
        bool ok = mbar_wait(&full[s], (tile / kTcStages) & 1);
        if (ok && tile >= 2) ok = mbar_wait(&acce[acc], ((tile >> 1) - 1) & 1);
        if (!ok || *reinterpret_cast<volatile uint32_t*>(abort_flag)) {
          if (!ok) {
            flag_status(a.status, TSD_DEV_TIMEOUT);
            atomicOr(abort_flag, 1u);
          }
          break;
        }
        tc_fence_after_sync();
        const uint32_t kb = smem_u32(stages + (size_t)s * kTcStageBytes);
        const uint32_t d = tmem + (uint32_t)(acc * 16);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t oa = (uint32_t)((ks >> 2) * (kTcTile * 128) + (ks & 3) * 32);
          const uint32_t ob = (uint32_t)((ks >> 2) * kQHalfBytes + (ks & 3) * 32);
          umma_bf16(d, sw128_desc(kb + oa, 1024), sw128_desc(qh + ob, 1024), idesc, ks > 0);
          if (QF32) umma_bf16(d, sw128_desc(kb + oa, 1024), sw128_desc(ql + ob, 1024), idesc, true);
        }
        umma_commit(&empty[s]);   // the stage may be refilled once these MMAs have read it
        umma_commit(&accf[acc]);  // the accumulator is ready
        issued = tile + 1;
      }
      // no MMA may be in flight when tensor memory is freed
      if (issued > 0 && !mbar_wait(&accf[(issued - 1) & 1], ((issued - 1) >> 1) & 1))
        flag_status(a.status, TSD_DEV_TIMEOUT);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;   // this warp's 32 tensor-memory lanes: tokens 32 q .. 32 q + 31
    for (int tile = 0; tile < ntiles; ++tile) {
      const int acc = tile & 1;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&accf[acc], (tile >> 1) & 1);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) flag_status(a.status, TSD_DEV_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      uint32_t r[16];
      tmem_ld16(tmem + (uint32_t)(acc * 16) + ((uint32_t)(32 * quarter) << 16), r);
      tmem_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[acc]);
      const int tok = tok0 + tile * kTcTile + kTcRowsPerQuarter * quarter + lane;
      if (lane < kTcRowsPerQuarter) {
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < nlists && tok < s_kvl[m]) a.scores[s_srow[m] + tok] = __uint_as_float(r[m]);
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTcCols);
  }
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

// Fast path for lists much longer than k: a threshold from a sample, then ONE pass over the
// scores.  Take a strided sample of the list (1024 scores, or 4096 from 64K scores on) and r,
// its expected count above the k-th score plus 4 standard deviations plus 4.  The sample's
// r-th largest key with its low 10 bits cleared (lo) has, with overwhelming probability, at
// least k scores at or above it.  One ordered pass copies every (index, key) with key >= lo
// into shared memory in index order; the exact radix select and the ordered output then run
// over those few thousand entries only.  Returns false, having written nothing, when the
// sample says too many keys would be kept or the pass kept more than fit or fewer than k: the
// caller then runs the full passes.
// The score of an order-preserving key (inverse of score_key; -0 comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

constexpr int kFastMinL = 4096;
constexpr int kFastSample = 1024;        // sampled scores, lists shorter than kFastLongL
constexpr int kFastSampleLong = 4096;    // the same from kFastLongL on: a tighter threshold
constexpr int kFastLongL = 65536;
constexpr int kFastCap = kCandMax / 2;   // kept entries: keys in cand[0, cap), indices in cand[cap, 2 cap)

__device__ bool select_fast(SelectSmem& S, const float* row, int L, int k, int32_t* out, float* osc, int k_max) {
  uint32_t* ckey = S.cand;
  uint32_t* cidx = S.cand + kFastCap;
  // ---- the r_lo-th largest of a strided sample of keys ----
  const int ns = L >= kFastLongL ? kFastSampleLong : kFastSample;
  const float mean = (float)ns * (float)k / (float)L;
  const int r_lo = (int)ceilf(mean + 4.f * sqrtf(mean) + 4.f);
  if (r_lo >= ns || (int64_t)r_lo * L > (int64_t)kFastCap * ns * 3 / 4) return false;
  for (int s = threadIdx.x; s < ns; s += kSelectThreads)
    ckey[s] = score_key(__ldcg(row + (int)(((int64_t)s * L) / ns)));
  // two 11-bit rounds: lo is the r_lo-th largest sampled key with its low 10 bits cleared,
  // which keeps a little more than the exact sample key would
  uint32_t prefix = 0u;
  int need = r_lo, shift = 32;
  while (shift > 10) {
    const int nb = 11;
    shift -= nb;
    const bool first = shift + nb == 32;
    for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[i] = 0u;
    __syncthreads();
    for (int c = threadIdx.x; c < ns; c += kSelectThreads) {
      const uint32_t key = ckey[c];
      if (first || (key >> (shift + nb)) == prefix) atomicAdd(&S.hist[(key >> shift) & ((1u << nb) - 1u)], 1u);
    }
    __syncthreads();
    select_bin(S, 1 << nb, need);
    prefix = (prefix << nb) | (uint32_t)S.found_bin;
    need -= S.found_above;
    __syncthreads();
  }
  const uint32_t lo_key = prefix << shift;

  // ---- one ordered pass: every key >= lo, in index order ----
  // The key map is monotone, so key >= lo is score >= lo_f, the score whose key is lo: the
  // pass compares floats and forms keys only for the entries it keeps.
  const float lo_f = key_score(lo_key);
  const int tile_elems = kSelectThreads * kSelPerThread;
  int kept = 0;
  for (int base = 0; base < L; base += tile_elems) {
    const int i0 = base + threadIdx.x * kSelPerThread;
    float f[kSelPerThread];
    load16(row, i0, L, f);
    uint32_t keep = 0u;
    if (base + tile_elems <= L) {   // a full tile (uniform over the block)
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j) keep |= (f[j] >= lo_f ? 1u : 0u) << j;
    } else {
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j) keep |= (i0 + j < L && f[j] >= lo_f ? 1u : 0u) << j;
    }
    int tot;
    int pos = kept + block_exclusive_scan<kSelectThreads>(__popc(keep), S.scan_tmp, &tot);
    if (keep != 0u) {
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j)
        if ((keep >> j) & 1u) {
          if (pos < kFastCap) {
            ckey[pos] = score_key(f[j]);
            cidx[pos] = (uint32_t)(i0 + j);
          }
          ++pos;
        }
    }
    kept += tot;
  }
  __syncthreads();
  if (kept > kFastCap || kept < k) return false;

  // ---- exact k-th key among the kept entries ----
  prefix = 0u;
  need = k;
  shift = 32;
  while (shift > 0) {
    const int nb = shift >= 11 ? 11 : shift;
    shift -= nb;
    const bool first = shift + nb == 32;
    for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[i] = 0u;
    __syncthreads();
    for (int c = threadIdx.x; c < kept; c += kSelectThreads) {
      const uint32_t key = ckey[c];
      if (first || (key >> (shift + nb)) == prefix) atomicAdd(&S.hist[(key >> shift) & ((1u << nb) - 1u)], 1u);
    }
    __syncthreads();
    select_bin(S, 1 << nb, need);
    prefix = (prefix << nb) | (uint32_t)S.found_bin;
    need -= S.found_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = need;

  // ---- ordered output over the kept entries ----
  constexpr int kPer = (kFastCap + kSelectThreads - 1) / kSelectThreads;
  const int c0 = threadIdx.x * kPer;
  int neq = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) neq += (c0 + j < kept && ckey[c0 + j] == T);
  int eq_total;
  int eq_run = block_exclusive_scan<kSelectThreads>(neq, S.scan_tmp, &eq_total);
  int nsel = 0;
  uint32_t selmask = 0u;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (c0 + j >= kept) break;
    const uint32_t key = ckey[c0 + j];
    bool sel = key > T;
    if (key == T) {
      sel = eq_run < need_eq;
      ++eq_run;
    }
    if (sel) {
      selmask |= 1u << j;
      ++nsel;
    }
  }
  int sel_total;
  int pos = block_exclusive_scan<kSelectThreads>(nsel, S.scan_tmp, &sel_total);
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (selmask & (1u << j)) {
      if (pos < k) {
        out[pos] = (int32_t)cidx[c0 + j];
        if (osc != nullptr) osc[pos] = key_score(ckey[c0 + j]);
      }
      ++pos;
    }
  for (int i = k + threadIdx.x; i < k_max; i += kSelectThreads) {
    out[i] = -1;
    if (osc != nullptr) osc[i] = -CUDART_INF_F;
  }
  return true;
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
  float* osc = a.out_scores != nullptr ? a.out_scores + (int64_t)th * a.k_max : nullptr;
  if (a.out_count != nullptr && threadIdx.x == 0) a.out_count[th] = k;
  const float* row = a.scores + (int64_t)th * a.score_stride;

  if (k == L || k == 0) {   // every visible token is kept, or none
    for (int i = threadIdx.x; i < a.k_max; i += kSelectThreads) {
      out[i] = i < k ? i : -1;
      if (osc != nullptr) osc[i] = i < k ? __ldcg(row + i) + 0.f : -CUDART_INF_F;
    }
    return;
  }
  if (L >= kFastMinL && select_fast(S, row, L, k, out, osc, a.k_max)) return;
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
  // (compared as floats: key > T is score > T_f and key == T is score == T_f, -0 == +0 included)
  const float T_f = key_score(T);
  int eq_before = 0, sel_before = 0;
  for (int base = 0; base < L; base += tile_elems) {
    const int i0 = base + threadIdx.x * kSelPerThread;
    float f[kSelPerThread];
    load16(row, i0, L, f);
    int neq = 0;
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j)
      if (i0 + j < L && f[j] == T_f) ++neq;
    int eq_total;
    int eq_run = eq_before + block_exclusive_scan<kSelectThreads>(neq, S.scan_tmp, &eq_total);
    int nsel = 0;
    uint32_t selmask = 0;
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j) {
      bool sel = false;
      if (i0 + j < L) {
        if (f[j] > T_f) sel = true;
        else if (f[j] == T_f) { sel = eq_run < need_eq; ++eq_run; }
      }
      if (sel) { selmask |= 1u << j; ++nsel; }
    }
    int sel_total;
    int pos = sel_before + block_exclusive_scan<kSelectThreads>(nsel, S.scan_tmp, &sel_total);
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j)
      if (selmask & (1u << j)) {
        if (pos < k) {
          out[pos] = i0 + j;
          if (osc != nullptr) osc[pos] = f[j] + 0.f;   // -0 as +0, like the key
        }
        ++pos;
      }
    eq_before += eq_total;
    sel_before += sel_total;
  }
  for (int i = k + threadIdx.x; i < a.k_max; i += kSelectThreads) {
    out[i] = -1;
    if (osc != nullptr) osc[i] = -CUDART_INF_F;
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// Which scoring kernel runs: the warp-level mma.sync kernel (default, the faster one on the
// measured workloads), or with TSD_SCORE_KERNEL=tcgen05 in the environment the tcgen05
// kernel.  Both use 5 CTAs per SM, so the window plan is the same.
static bool score_on_tcgen05() {
  const char* e = getenv("TSD_SCORE_KERNEL");
  return e != nullptr && strcmp(e, "tcgen05") == 0;
}

cudaError_t launch_topk(const TopkArgs& a, const KvMaps& maps, int nwin, int batch, int hkv, int num_lists,
                        cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_score_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ScLayout<false, kScStages>::bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_score_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)ScLayout<true, kScStages>::bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_score_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)TcLayout<false>::bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_score_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)TcLayout<true>::bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SelectSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 g1(nwin, hkv * a.list_groups, batch);
  if (score_on_tcgen05()) {
    if (a.qv.q_f32) {
      topk_score_tc_kernel<true><<<g1, kTcThreads, TcLayout<true>::bytes, stream>>>(a, maps);
    } else {
      topk_score_tc_kernel<false><<<g1, kTcThreads, TcLayout<false>::bytes, stream>>>(a, maps);
    }
  } else if (a.qv.q_f32) {
    topk_score_kernel<true><<<g1, kScThreads, ScLayout<true, kScStages>::bytes, stream>>>(a, maps);
  } else {
    topk_score_kernel<false><<<g1, kScThreads, ScLayout<false, kScStages>::bytes, stream>>>(a, maps);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<num_lists, kSelectThreads, sizeof(SelectSmem), stream>>>(a);
  return cudaGetLastError();
}

// The selection alone, over scores another kernel wrote into the workspace (the label indexer).
cudaError_t launch_topk_select_only(const TopkArgs& a, int num_lists, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e =
        cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SelectSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  topk_select_kernel<<<num_lists, kSelectThreads, sizeof(SelectSmem), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tsd
