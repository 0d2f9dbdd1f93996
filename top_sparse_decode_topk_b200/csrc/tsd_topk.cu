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
#include "tsd_filter.cuh"
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
// 6 CTAs per SM with bf16 queries (measured on the ragged batch's filtered scoring: 882 against
// 930 us at 5); fp32 queries carry a second query tile and fit 5
static_assert(ScLayout<false, kScStages>::bytes + 1024 <= 228 * 1024 / kScCtasPerSm, "scoring CTAs per SM");
static_assert(ScLayout<true, kScStages>::bytes + 1024 <= 228 * 1024 / 5, "scoring CTAs per SM, fp32 queries");

// Candidate slots a quad reserves at a time, and the index that marks a reserved slot left unused.
constexpr uint32_t kCandChunk = 8;
constexpr uint32_t kCandHole = 0xFFFFFFFFu;

template <bool QF32>
__global__ void __launch_bounds__(kScThreads, QF32 ? 5 : kScCtasPerSm) topk_score_kernel(TopkArgs a, const __grid_constant__ KvMaps maps) {
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
  const int tok0 = win * a.window;
  const int tok_end = min(tok0 + a.window, si.len);
  const bool idle = nlists <= 0 || tok_end <= tok0;
  // Under the filter the kernels after this one read what the pre-pass wrote once this grid has
  // completed, so every CTA waits for the pre-pass before it exits (the consumers below do).
  if (idle) {
    if (a.filter) pdl_wait();
    return;
  }
  const int ntiles = (tok_end - tok0 + kTileTok - 1) / kTileTok;
  const bool use_tma = a.kv.page_table == nullptr || a.kv.page_shift >= 3;
  if (smem_u32(stages) & 1023u) {
    if (threadIdx.x == 0) flag_status(a.status, TSD_DEV_TIMEOUT);
    if (a.filter) pdl_wait();
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
  pdl_launch_dependents();   // the selection may launch; it waits for this kernel's scores

  if (warp == kScConsumers) {
    produce_tiles<kScStages, kTileBytesKV, false>(a.kv, maps, b, g, tok0, tok_end, ntiles, stages, full,
                                                  empty, abort_flag, use_tma, lane, a.status);
    return;
  }
  // this lane's query rows m = lane/4 and lane/4 + 8: visible length and score row
  int kvl[2];
  float* srow[2];
  float* prow[2];   // the list's sample row: the score of every 2^sample_shift-th token
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int m = (lane >> 2) + 8 * hr;
    kvl[hr] = 0;
    srow[hr] = a.scores;
    prow[hr] = a.samples;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int j = mg / G;
      kvl[hr] = min(kv_len_of(a.qv, si, j), tok_end);
      const int64_t list = (int64_t)(si.t0 + j) * a.qv.hq + g * G + (mg - j * G);
      srow[hr] = a.scores + list * a.score_stride;
      prow[hr] = a.samples + list * a.sample_stride;
    }
  }
  const int smask = (1 << a.sample_shift) - 1;
  // candidate filter: this lane's lists' thresholds and candidate buffers.  A score is appended
  // unless it is below lo_f, the float whose key is lo: every score whose key reaches lo, plus
  // NaNs whatever their key (the selection drops the keys below lo).
  float lo_f[2] = {CUDART_INF_F, CUDART_INF_F};
  uint32_t* ccnt[2] = {nullptr, nullptr};
  uint2* cbuf[2] = {nullptr, nullptr};
  uint32_t pool_next[2] = {0u, 0u}, pool_end[2] = {0u, 0u};   // the quad's reserved, unused slots
  if (a.filter) {
    pdl_wait();   // the pre-pass wrote lo
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = (lane >> 2) + 8 * hr;
      if (m < nlists) {
        const int mg = lg * a.lists_per_cta + m;
        const int j = mg / G;
        const int64_t list = (int64_t)(si.t0 + j) * a.qv.hq + g * G + (mg - j * G);
        const uint32_t lo = __ldcg(a.lo_key + list);
        // keys above +inf's are positive NaNs, keys below -inf's negative ones
        lo_f[hr] = lo >= 0xFF800000u ? CUDART_INF_F : (lo <= 0x007FFFFFu ? -CUDART_INF_F : key_score(lo));
        ccnt[hr] = a.cand_cnt + list;
        cbuf[hr] = a.cand + list * kTopkCandCap;
      }
    }
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    if (!consume_wait<kScStages>(full, abort_flag, tile, lane, a.status)) break;
    float sc[2][4];
    qk_tile<QF32, true>(qhi, qlo, stages + (size_t)(tile % kScStages) * kTileBytesKV, warp, lane, sc);
    // the fragments are in registers: release the stage to the producer before the stores
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[tile % kScStages]);
    const int tbase = tok0 + tile * kTileTok + 16 * warp + 2 * (lane & 3);
    if (!a.filter) {
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
          if ((tk & smask) == 0 && tk < kvl[hr]) prow[hr][tk >> a.sample_shift] = sc[nt][2 * hr];
        }
      continue;
    }
    // the filtered form: the lane's scores whose keys reach its lists' thresholds go to the lists'
    // candidate buffers.  The 4 lanes of a quad share a list row and take their slots, in lane
    // order, from the quad's pool; the last lane refills the pool kCandChunk slots at a time with
    // one atomic on the list's counter, so that the round trip is rare.
    uint32_t f[2] = {0u, 0u};
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
#pragma unroll
      for (int e = 0; e < 4; ++e) f[hr] |= (uint32_t)!(sc[e >> 1][2 * hr + (e & 1)] < lo_f[hr]) << e;
      if (tbase + 9 >= kvl[hr]) {   // the tile's tail: drop the tokens at or past kv_len
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (tbase + 8 * (e >> 1) + (e & 1) >= kvl[hr]) f[hr] &= ~(1u << e);
      }
    }
    if (__ballot_sync(0xFFFFFFFFu, (f[0] | f[1]) != 0u) == 0u) continue;
    // both rows' counts in one word: inclusive prefix over the quad, and the quad's totals
    const uint32_t cpk = (uint32_t)__popc(f[0]) | ((uint32_t)__popc(f[1]) << 16);
    uint32_t x = cpk;
    uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, 1);
    if ((lane & 3) >= 1) x += y;
    y = __shfl_up_sync(0xFFFFFFFFu, x, 2);
    if ((lane & 3) >= 2) x += y;
    const uint32_t tpk = __shfl_sync(0xFFFFFFFFu, x, lane | 3);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const uint32_t tot = (tpk >> (16 * hr)) & 0xFFFFu;
      const uint32_t room = pool_end[hr] - pool_next[hr];
      const bool grow = tot > room;   // the same in the quad's 4 lanes
      uint32_t fresh = 0u, want = 0u;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        if (grow) {
          want = (tot - room + kCandChunk - 1) / kCandChunk * kCandChunk;
          if ((lane & 3) == 3) fresh = atomicAdd(ccnt[hr], want);
        }
        fresh = __shfl_sync(0xFFFFFFFFu, fresh, lane | 3);
      }
      uint32_t i = ((x >> (16 * hr)) & 0xFFFFu) - ((cpk >> (16 * hr)) & 0xFFFFu);   // first rank in the quad
      uint32_t bits = f[hr];
      while (bits != 0u) {
        const int e = __ffs(bits) - 1;
        bits &= bits - 1u;
        const uint32_t slot = i < room ? pool_next[hr] + i : fresh + (i - room);
        const float v = e == 0 ? sc[0][2 * hr] : (e == 1 ? sc[0][2 * hr + 1] : (e == 2 ? sc[1][2 * hr] : sc[1][2 * hr + 1]));
        if (slot < (uint32_t)kTopkCandCap)
          cbuf[hr][slot] = make_uint2(score_key(v), (uint32_t)(tbase + 8 * (e >> 1) + (e & 1)));
        ++i;
      }
      if (grow) {
        pool_next[hr] = fresh + (tot - room);
        pool_end[hr] = fresh + want;
      } else {
        pool_next[hr] += tot;
      }
    }
  }
  if (a.filter && (lane & 3) == 3) {
    // the pools' unused slots become holes: an index no list has, which the selection skips
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
      for (uint32_t slot = pool_next[hr]; slot < pool_end[hr] && slot < (uint32_t)kTopkCandCap; ++slot)
        cbuf[hr][slot] = make_uint2(0u, kCandHole);
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
static_assert(TcLayout<false>::bytes + 1024 <= 228 * 1024 / kTcCtasPerSm, "tensor-core scoring CTAs per SM");

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
          if (m < nlists && tok < s_kvl[m]) {
            a.scores[s_srow[m] + tok] = __uint_as_float(r[m]);
            if ((tok & ((1 << a.sample_shift) - 1)) == 0)
              a.samples[s_srow[m] / a.score_stride * a.sample_stride + (tok >> a.sample_shift)] = __uint_as_float(r[m]);
          }
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

// Sequence b, visible length L and kept count k = min(k_t, L) of list th (token t = th / Hq).
__device__ __forceinline__ void list_len_k(const TopkArgs& a, int th, int& b, int& L, int& k) {
  const int t = th / a.qv.hq;
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
  L = 0;
  if (t >= si.t0 && t < si.t0 + si.n) L = kv_len_of(a.qv, si, t - si.t0);
  int kreq = a.k_max;
  if (a.k_per_token != nullptr) {
    kreq = __ldg(a.k_per_token + t);
    kreq = kreq < 0 ? 0 : (kreq > a.k_max ? a.k_max : kreq);
  }
  k = kreq < L ? kreq : L;
}
__device__ __forceinline__ void list_len_k(const TopkArgs& a, int th, int& L, int& k) {
  int b;
  list_len_k(a, th, b, L, k);
}

// ---------------------------------------------------------------------------
// Candidate filter of the exact indexer: the pre-pass
// ---------------------------------------------------------------------------
// Before the scoring kernel, topk_prepass_kernel scores every 2^sample_shift-th token of every
// list (bf16 queries) and turns each list's sample into a threshold key lo, as the selection's
// sampled fast path would.  The scoring kernel then appends every score whose key reaches lo to
// the list's candidate buffer instead of writing the score row, and the selection works on the
// candidates alone (see topk_cand_kernel).
//
// Grid (splits, Hkv x list groups, batch), kPpWarps warps per CTA.  The splits of a (sequence,
// kv head, list group) share its sample tiles; each writes its samples, and the last to arrive
// on the group's counter -- the candidate counter of the group's first list, which the scoring
// kernel needs zero only after this kernel has completed -- computes the group's thresholds
// and leaves the counter zero.
constexpr int kPpWarps = 8;

__global__ void __launch_bounds__(32 * kPpWarps, 2) topk_prepass_kernel(TopkArgs a) {
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();   // the scoring kernel may launch; its consumers wait for this grid
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, false);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;   // the same in every split of the group: no thresholds to make
  const int shift = a.sample_shift;
  const int64_t max_ns = ((int64_t)a.kv.max_seq_len + (1 << shift) - 1) >> shift;
  const int per_split = (int)(((max_ns + 15) / 16 + gridDim.x - 1) / gridDim.x);   // 16-row tiles
  const int ns_seq = (int)(((int64_t)si.len + (1 << shift) - 1) >> shift);
  const int tile_end = min((int)blockIdx.x * per_split + per_split, (ns_seq + 15) / 16);
  const int tr = lane >> 2, kq = 2 * (lane & 3);
  // B operand (q, bf16): lists 8 grp + tr, dims [16 ks + kq, +1] and [+8, +9]
  uint32_t bq[2][8][2];
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    const int m = 8 * grp + tr;
    const uint32_t* qrow = nullptr;
    if (m < nlists) {
      const int mg = lg * a.lists_per_cta + m;
      const int jt = mg / G;
      qrow = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(a.qv.q) +
                                               ((int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G)) * kHeadDim);
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      bq[grp][ks][0] = qrow != nullptr ? __ldg(qrow + 8 * ks + kq / 2) : 0u;
      bq[grp][ks][1] = qrow != nullptr ? __ldg(qrow + 8 * ks + kq / 2 + 4) : 0u;
    }
  }
  // the two sample rows of this lane in tile t (A rows tr and tr + 8); a bad page is flagged
  auto rows_of = [&](int t, uint32_t* rr) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t tok = (int64_t)(t * 16 + tr + 8 * h) << shift;
      rr[h] = t < tile_end && tok < si.len ? kv_row(a.kv, b, g, (int)tok) : kInvalidRow;
      if (t < tile_end && tok < si.len && rr[h] == kInvalidRow) flag_status(a.status, TSD_DEV_BAD_PAGE);
    }
  };
  uint32_t rnext[2];
  rows_of((int)blockIdx.x * per_split + warp, rnext);
  for (int tile = (int)blockIdx.x * per_split + warp; tile < tile_end; tile += kPpWarps) {
    const int j0 = tile * 16;
    const uint32_t rr[2] = {rnext[0], rnext[1]};
    rows_of(tile + kPpWarps, rnext);   // the next tile's page lookups overlap this tile's loads
    uint32_t af[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(a.kv.k + (int64_t)(rr[h] != kInvalidRow ? rr[h] : 0) * kHeadDim);
        af[ks][h] = rr[h] != kInvalidRow ? __ldg(kr + 8 * ks + kq / 2) : 0u;
        af[ks][2 + h] = rr[h] != kInvalidRow ? __ldg(kr + 8 * ks + kq / 2 + 4) : 0u;
      }
    }
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      if (8 * grp >= nlists) break;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_bf16(d, af[ks], bq[grp][ks][0], bq[grp][ks][1]);
      // D: (row tr, lists 8 grp + kq, + 1) = d0, d1; (row tr + 8, the same lists) = d2, d3
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int m = 8 * grp + kq + u;
        if (m >= nlists) continue;
        const int mg = lg * a.lists_per_cta + m;
        const int jt = mg / G;
        const int kvl = kv_len_of(a.qv, si, jt);
        float* prow = a.samples + ((int64_t)(si.t0 + jt) * a.qv.hq + g * G + (mg - jt * G)) * a.sample_stride;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = j0 + tr + 8 * h;
          if (rr[h] != kInvalidRow && ((int64_t)j << shift) < kvl) prow[j] = d[2 * h + u];
        }
      }
    }
  }
  // arrive; the last split of the group makes its thresholds
  const int j_first = (lg * a.lists_per_cta) / G;
  const int64_t first_list = (int64_t)(si.t0 + j_first) * a.qv.hq + g * G + (lg * a.lists_per_cta - j_first * G);
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(a.cand_cnt + first_list, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) a.cand_cnt[first_list] = 0u;
  for (int m = warp; m < nlists; m += kPpWarps) {
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
// ---------------------------------------------------------------------------
// Selection
// ---------------------------------------------------------------------------
constexpr int kSelWarps = kSelectThreads / 32;

constexpr int kSelMaskIters = 16;   // segment steps whose keep masks the fast path keeps (L <= 128K)

struct SelectSmem {
  uint32_t hist[2][kSelBins];   // the fast path alternates; the multi-pass path uses hist[0]
  uint32_t cand[kCandMax];
  uint16_t keep[kSelWarps][kSelMaskIters][32];   // fast path: each lane's keep bits of each step
  int scan_tmp[kSelWarps + 1];
  int found_bin, found_above, ncand;
  int wcount[kSelWarps];
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
    if (bin >= 0) local += (int)S.hist[0][bin];
  }
  int total;
  int run = block_exclusive_scan<kSelectThreads>(local, S.scan_tmp, &total);
  for (int j = 0; j < per; ++j) {
    const int bin = hi - 1 - j;
    if (bin < 0) break;
    const int c = (int)S.hist[0][bin];
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

// Warp 0 only: in hist[0, nb) find the bin d (scanning from the top) with count(bins above d)
// < need <= count(bins >= d); lane 0 writes S.found_bin and S.found_above.  Lane l first sums
// the contiguous bins [nb - (l + 1) per, nb - l per), read in a rotated order so that the 32
// lanes hit 32 different banks; a lane scan finds the lane whose range crosses `need`, and
// the 32 lanes then split that range (per / 32 bins each) for a second scan.
template <class SM>
__device__ __forceinline__ void warp_find_bin(SM& S, const uint32_t* hist, int nb, int need) {
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int per = nb >> 5;
  int sum = 0;
  {
    const int hi = nb - lane * per;
    for (int j = 0; j < per; ++j) sum += (int)hist[hi - 1 - ((j + lane) & (per - 1))];
  }
  int inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, inc, o);
    if (lane >= o) inc += y;
  }
  const unsigned cross = __ballot_sync(FULL, inc - sum < need && need <= inc);
  if (cross == 0u) {   // only for inconsistent counts
    if (lane == 0) {
      S.found_bin = 0;
      S.found_above = 0;
    }
    return;
  }
  const int cl = __ffs(cross) - 1;
  const int base_above = __shfl_sync(FULL, inc - sum, cl);
  const int top = nb - cl * per;        // the crossing lane's bins are [top - per, top)
  const int q = per >> 5;               // bins per lane in the second step (1 or 2)
  int s2 = 0;
  for (int t = 0; t < q; ++t) s2 += (int)hist[top - 1 - (lane * q + t)];
  int inc2 = s2;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, inc2, o);
    if (lane >= o) inc2 += y;
  }
  const int ex2 = base_above + inc2 - s2;
  const unsigned c2 = __ballot_sync(FULL, ex2 < need && need <= base_above + inc2);
  const int l2 = c2 ? __ffs(c2) - 1 : 0;
  if (lane == l2) {
    int run = ex2, bin = top - 1 - lane * q;
    for (int t = 0; t < q; ++t) {
      const int b = top - 1 - (lane * q + t);
      const int c = (int)hist[b];
      bin = b;
      if (run + c >= need) break;
      run += c;
    }
    S.found_bin = bin;
    S.found_above = run;
  }
}

// One radix round over keys[0, n) in shared memory: histogram of the nb-bit digit at `shift`
// of the keys whose higher bits equal `prefix` (every key when `first`) into hist[cur], while
// hist[cur ^ 1] is zeroed for the next round; then warp 0 finds the digit holding the
// need-th largest key.  hist[cur] must be zero on entry.  Two block barriers.
__device__ __forceinline__ void radix_round(SelectSmem& S, const uint32_t* keys, int n, int nb, int shift, bool first,
                                            uint32_t prefix, int need, int cur) {
  uint32_t* h = S.hist[cur];
  uint32_t* z = S.hist[cur ^ 1];
  for (int i = threadIdx.x; i < kSelBins; i += kSelectThreads) z[i] = 0u;
  const uint32_t mask = (1u << nb) - 1u;
  for (int c = threadIdx.x; c < n; c += kSelectThreads) {
    const uint32_t key = keys[c];
    if (first || (key >> (shift + nb)) == prefix) atomicAdd(&h[(key >> shift) & mask], 1u);
  }
  __syncthreads();
  if (threadIdx.x < 32) warp_find_bin(S, h, 1 << nb, need);
  __syncthreads();
}

constexpr int kFastMinL = 4096;
constexpr int kFastCap = kCandMax / 2;   // kept entries: keys in cand[0, cap), indices in cand[cap, 2 cap)
constexpr int kFastUnroll = 4;           // float4 loads in flight per lane in the segment passes

// Fast path for lists much longer than k: a threshold from a sample, then the scores at or
// above it, then the exact selection among those few.
//  1. The list's strided sample -- every 2^sample_shift-th score (every 32nd up to 128K tokens),
//     written by the scoring kernel into a compact row and read here contiguously -- and r,
//     its expected count above the k-th score plus 4 standard deviations plus 4.  Two radix
//     rounds give the sample's r-th largest key with its low 10 bits cleared (lo), which has,
//     with overwhelming probability, at least k scores at or above it.  The result does not
//     depend on the sample: whatever lo is, at least k kept scores means every top-k score is
//     kept, and fewer means the fallback below.
//  2. Every warp owns a contiguous segment of the list: it counts its scores >= lo, the
//     counts give every warp its output offset, and it copies its (key, index) pairs in index
//     order (ballot and lane scan) -- a second read of the segment, from L2.  One barrier
//     orders the whole list, where a block-wide scan per tile took three.
//  3. Three radix rounds among the kept keys give the exact k-th key T and how many keys equal
//     to T are kept; keys > T and the lowest-index keys == T are written in index order.
// Each radix digit is found by one warp, on histograms that alternate between two buffers.
// Returns false, having written nothing, when the sample says too many keys would be kept or
// the segments hold more than fit or fewer than k: the caller then runs the multi-pass path.
__device__ bool select_fast(SelectSmem& S, const float* row, const float* samp, int sample_shift, int L, int k,
                            int32_t* out, float* osc, int k_max) {
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* ckey = S.cand;
  uint32_t* cidx = S.cand + kFastCap;
  // ---- 1. the threshold lo from a strided sample ----
  // the scoring kernel wrote every 2^sample_shift-th score of the list to its sample row
  const int ns = (L + (1 << sample_shift) - 1) >> sample_shift;
  const float mean = (float)ns * (float)k / (float)L;
  const int r_lo = (int)ceilf(mean + 4.f * sqrtf(mean) + 4.f);
  if (ns > kFastCap || r_lo >= ns || (int64_t)r_lo * L > (int64_t)kFastCap * ns * 3 / 4) return false;
  for (int i = threadIdx.x; i < kSelBins; i += kSelectThreads) S.hist[0][i] = 0u;
  for (int s = threadIdx.x; s < ns; s += kSelectThreads) ckey[s] = score_key(__ldcg(samp + s));
  __syncthreads();
  radix_round(S, ckey, ns, 11, 21, true, 0u, r_lo, 0);
  uint32_t prefix = (uint32_t)S.found_bin;
  int need = r_lo - S.found_above;
  radix_round(S, ckey, ns, 11, 10, false, prefix, need, 1);
  prefix = (prefix << 11) | (uint32_t)S.found_bin;
  const float lo_f = key_score(prefix << 10);   // key >= lo  <=>  score >= lo_f (the map is monotone)

  // ---- 2. the scores >= lo, in index order ----
  // Each step a warp reads kRow * kFastUnroll scores: lane l the float4s at base + kRow u + 4 l.
  // The counting pass keeps every lane's keep bits of every step (16 bits: float4 u, element j
  // at bit 4 u + j) when the segment has at most kSelMaskIters steps, so that the copying pass
  // skips the steps where the warp keeps nothing and visits only the kept elements.
  constexpr int kRow = 128;
  constexpr int kStep = kRow * kFastUnroll;
  const int seg = ((L + kSelWarps - 1) / kSelWarps + kRow - 1) / kRow * kRow;
  const int s0 = min(warp * seg, L), s1 = min(s0 + seg, L);
  const bool masks = (seg + kStep - 1) / kStep <= kSelMaskIters;
  auto keep_bits = [&](const float4* v, int base) -> uint32_t {
    uint32_t m = 0u;
    if (base + kStep <= s1) {   // a whole step inside the segment (uniform over the warp)
#pragma unroll
      for (int u = 0; u < kFastUnroll; ++u)
        m |= ((uint32_t)(v[u].x >= lo_f) | ((uint32_t)(v[u].y >= lo_f) << 1) | ((uint32_t)(v[u].z >= lo_f) << 2) |
              ((uint32_t)(v[u].w >= lo_f) << 3)) << (4 * u);
    } else {
#pragma unroll
      for (int u = 0; u < kFastUnroll; ++u) {
        const int i = base + kRow * u + 4 * lane;
        m |= ((uint32_t)(i < s1 && v[u].x >= lo_f) | ((uint32_t)(i + 1 < s1 && v[u].y >= lo_f) << 1) |
              ((uint32_t)(i + 2 < s1 && v[u].z >= lo_f) << 2) | ((uint32_t)(i + 3 < s1 && v[u].w >= lo_f) << 3))
             << (4 * u);
      }
    }
    return m;
  };
  auto load_step = [&](float4* v, int base) {
#pragma unroll
    for (int u = 0; u < kFastUnroll; ++u) {
      const int i = base + kRow * u + 4 * lane;
      v[u] = i < s1 ? __ldcg(reinterpret_cast<const float4*>(row + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  int cnt = 0;
  for (int base = s0, it = 0; base < s1; base += kStep, ++it) {
    float4 v[kFastUnroll];
    load_step(v, base);
    const uint32_t m = keep_bits(v, base);
    cnt += __popc(m);
    if (masks) S.keep[warp][it][lane] = (uint16_t)m;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o);
  if (lane == 0) S.wcount[warp] = cnt;
  __syncthreads();
  int off = 0, kept = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const int c = S.wcount[w];
    off += w < warp ? c : 0;
    kept += c;
  }
  if (kept > kFastCap || kept < k) return false;   // the same decision in every thread
  static_assert(kFastUnroll <= 4, "one 8-bit count field per float4 in a 32-bit word");
  for (int base = s0, it = 0; base < s1; base += kStep, ++it) {
    uint32_t m;
    float4 v[kFastUnroll];
    if (masks) {
      m = S.keep[warp][it][lane];
      if (__ballot_sync(FULL, m != 0u) == 0u) continue;   // nothing kept in this step
      load_step(v, base);
    } else {
      load_step(v, base);
      m = keep_bits(v, base);
    }
    // the kept counts of the lane's float4s (each <= 4) packed 8 bits apart: one lane scan gives
    // every float4's output offset (a field's warp total is at most 128)
    uint32_t packed = 0u;
#pragma unroll
    for (int u = 0; u < kFastUnroll; ++u) packed |= (uint32_t)__popc((m >> (4 * u)) & 0xFu) << (8 * u);
    uint32_t inc = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(FULL, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t excl = inc - packed, tot = __shfl_sync(FULL, inc, 31);
#pragma unroll
    for (int u = 0; u < kFastUnroll; ++u) {
      int pos = off + (int)((excl >> (8 * u)) & 0xFFu);
      uint32_t nib = (m >> (4 * u)) & 0xFu;
      const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      while (nib != 0u) {
        const int j = __ffs(nib) - 1;
        nib &= nib - 1u;
        float x = f[0];
        x = j == 1 ? f[1] : x;
        x = j == 2 ? f[2] : x;
        x = j == 3 ? f[3] : x;
        ckey[pos] = score_key(x);
        cidx[pos] = (uint32_t)(base + kRow * u + 4 * lane + j);
        ++pos;
      }
      off += (int)((tot >> (8 * u)) & 0xFFu);
    }
  }
  __syncthreads();

  // ---- 3. the exact k-th key among the kept ones, then the ordered output ----
  radix_round(S, ckey, kept, 11, 21, true, 0u, k, 0);
  prefix = (uint32_t)S.found_bin;
  need = k - S.found_above;
  radix_round(S, ckey, kept, 11, 10, false, prefix, need, 1);
  prefix = (prefix << 11) | (uint32_t)S.found_bin;
  need -= S.found_above;
  radix_round(S, ckey, kept, 10, 0, false, prefix, need, 0);
  const uint32_t T = (prefix << 10) | (uint32_t)S.found_bin;
  const int need_eq = need - S.found_above;   // keys == T to keep: the lowest-index ones

  // warp w takes the kept entries [r0, r1); its lanes walk them 32 at a time
  const int R = (kept + kSelWarps - 1) / kSelWarps;
  const int r0 = min(warp * R, kept), r1 = min(r0 + R, kept);
  int neq = 0;
  for (int c = r0 + lane; c < r1; c += 32) neq += ckey[c] == T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) neq += __shfl_xor_sync(FULL, neq, o);
  if (lane == 0) S.wcount[warp] = neq;
  __syncthreads();
  int eq_before = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) eq_before += w < warp ? S.wcount[w] : 0;
  const unsigned below = (1u << lane) - 1u;
  int nsel = 0, eq_run = eq_before;
  for (int c0 = r0; c0 < r1; c0 += 32) {
    const int c = c0 + lane;
    const uint32_t key = c < r1 ? ckey[c] : 0u;
    const bool eq = c < r1 && key == T;
    const unsigned eqm = __ballot_sync(FULL, eq);
    const bool sel = c < r1 && (key > T || (eq && eq_run + __popc(eqm & below) < need_eq));
    nsel += __popc(__ballot_sync(FULL, sel));
    eq_run += __popc(eqm);
  }
  __syncthreads();   // every warp has read the equal-key counts
  if (lane == 0) S.wcount[warp] = nsel;
  __syncthreads();
  int pos = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) pos += w < warp ? S.wcount[w] : 0;
  eq_run = eq_before;
  for (int c0 = r0; c0 < r1; c0 += 32) {
    const int c = c0 + lane;
    const uint32_t key = c < r1 ? ckey[c] : 0u;
    const bool eq = c < r1 && key == T;
    const unsigned eqm = __ballot_sync(FULL, eq);
    const bool sel = c < r1 && (key > T || (eq && eq_run + __popc(eqm & below) < need_eq));
    const unsigned selm = __ballot_sync(FULL, sel);
    const int p = pos + __popc(selm & below);
    if (sel && p < k) {
      out[p] = (int32_t)cidx[c];
      if (osc != nullptr) osc[p] = key_score(key);
    }
    pos += __popc(selm);
    eq_run += __popc(eqm);
  }
  for (int i = k + threadIdx.x; i < k_max; i += kSelectThreads) {
    out[i] = -1;
    if (osc != nullptr) osc[i] = -CUDART_INF_F;
  }
  return true;
}

// ---------------------------------------------------------------------------
// The candidate path of the filtered indexer (topk_cand_kernel)
// ---------------------------------------------------------------------------
// One CTA per list.  The scoring kernel appended, in no particular order, the
// (key, index) of every score not below the list's threshold into `slots` reserved slots (at
// most kTopkCandCap), some of them holes; the keys below lo (NaN scores) and the holes are
// skipped here.  With at least k valid candidates they hold the whole top-k and every score
// equal to the k-th.  Three radix rounds over the candidates, read from L2 each time, give the
// k-th key T and the number need_eq of keys equal to T to keep.  Keys > T are marked in a bitmap
// of the list's tokens and keys == T in a second one; warp-owned word ranges, read 32 words at a
// time, give the tie ranks (the need_eq lowest-index ties are kept) and the output ranks, and
// the kept indices are written in ascending order.  A list with fewer than k valid candidates, or
// more than fit, goes into the queue that topk_select_kernel works off over recomputed rows.
constexpr int kCandBitmapTokens = kTopkCandMaxLen;   // longest list the bitmaps cover
constexpr int kCsUnroll = 8;                  // candidate loads in flight per thread
template <int NT>
struct CandSmem {
  uint32_t hist[2][kSelBins];               // radix histograms; after the rounds, the tie bitmap
  uint32_t above[kCandBitmapTokens / 32];   // keys > T
  int scan_tmp[NT / 32 + 1];   // block scans; the warps' counts of keys > T in the ordered output
  int warp_ties[NT / 32];       // the warps' counts of keys == T in the ordered output
  int found_bin, found_above, nvalid, slots;
};
static_assert(kCandBitmapTokens <= 2 * kSelBins * 32, "the tie bitmap reuses both histograms");
static_assert(sizeof(CandSmem<1024>) <= 48 * 1024, "static shared memory of the candidate kernel");

// Every valid candidate of the list (index < L, key >= lo) through f(key, index), kCsUnroll
// loads in flight per thread.
template <int NT, class F>
__device__ __forceinline__ void for_candidates(const uint2* cand, int slots, uint32_t L, uint32_t lo, F f) {
  for (int i0 = threadIdx.x; i0 < slots; i0 += NT * kCsUnroll) {
    uint2 v[kCsUnroll];
#pragma unroll
    for (int u = 0; u < kCsUnroll; ++u) {
      const int i = i0 + u * NT;
      v[u] = i < slots ? __ldcg(cand + i) : make_uint2(0u, kCandHole);
    }
#pragma unroll
    for (int u = 0; u < kCsUnroll; ++u)
      if (v[u].y < L && v[u].x >= lo) f(v[u].x, v[u].y);
  }
}

// One radix round over the valid candidates: histogram of digit (key >> shift) & (2^nb - 1)
// among the keys whose bits above shift + nb equal prefix, then the digit of the need-th
// largest.  Histograms alternate between S.hist[cur] and S.hist[cur ^ 1].
template <int NT>
__device__ void cand_round(CandSmem<NT>& S, const uint2* cand, int slots, uint32_t L, uint32_t lo, int nb, int shift,
                           uint32_t prefix, int need, int cur) {
  uint32_t* h = S.hist[cur];
  uint32_t* z = S.hist[cur ^ 1];
  for (int i = threadIdx.x; i < kSelBins; i += NT) z[i] = 0u;
  const uint32_t mask = (1u << nb) - 1u;
  for_candidates<NT>(cand, slots, L, lo, [&](uint32_t key, uint32_t) {
    if ((key >> (shift + nb)) == prefix) atomicAdd(&h[(key >> shift) & mask], 1u);
  });
  __syncthreads();
  if (threadIdx.x < 32) warp_find_bin(S, h, 1 << nb, need);
  __syncthreads();
}

// NT threads per list: 1024 when the lists are few enough for one wave, else 256.
template <int NT>
__global__ void __launch_bounds__(NT) topk_cand_kernel(TopkArgs a) {
  __shared__ CandSmem<NT> S;
  const int th = blockIdx.x;
  pdl_wait();   // the scoring kernel (and before it the pre-pass) has completed
  pdl_launch_dependents();
  const int2 m = __ldcg(a.meta + th);
  const uint32_t L = (uint32_t)m.x;
  const int k = m.y < a.k_max ? m.y : a.k_max;
  int32_t* out = a.out_idx + (int64_t)th * a.k_max;
  if (threadIdx.x == 0) {
    if (a.out_count != nullptr) a.out_count[th] = k;
    S.slots = (int)a.cand_cnt[th];
    a.cand_cnt[th] = 0u;   // zero again for the next call
    S.nvalid = 0;
  }
  if (k == 0 || k == (int)L) {   // every visible token is kept, or none
    for (int i = threadIdx.x; i < a.k_max; i += NT) out[i] = i < k ? i : -1;
    return;
  }
  const uint32_t lo = __ldcg(a.lo_key + th);
  const int words = (int)((L + 31) >> 5);
  for (int i = threadIdx.x; i < kSelBins; i += NT) {
    S.hist[0][i] = 0u;
    S.hist[1][i] = 0u;
  }
  for (int i = threadIdx.x; i < words && i < kCandBitmapTokens / 32; i += NT) S.above[i] = 0u;
  __syncthreads();
  const int slots = S.slots;
  if (slots < k || slots > kTopkCandCap || L > (uint32_t)kCandBitmapTokens) {
    if (threadIdx.x == 0) a.queue[atomicAdd(a.queue_cnt, 1u)] = th;
    return;
  }
  const uint2* cand = a.cand + (int64_t)th * kTopkCandCap;
  // the first radix round (top 11 key bits), counting the valid candidates on the way
  int mine = 0;
  for_candidates<NT>(cand, slots, L, lo, [&](uint32_t key, uint32_t) {
    atomicAdd(&S.hist[0][key >> 21], 1u);
    ++mine;
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xFFFFFFFFu, mine, o);
  if ((threadIdx.x & 31) == 0 && mine != 0) atomicAdd(&S.nvalid, mine);
  __syncthreads();
  if (S.nvalid < k) {   // the same in every thread; nothing was written
    if (threadIdx.x == 0) a.queue[atomicAdd(a.queue_cnt, 1u)] = th;
    return;
  }
  if (threadIdx.x < 32) warp_find_bin(S, S.hist[0], kSelBins, k);
  __syncthreads();
  uint32_t prefix = (uint32_t)S.found_bin;
  int need = k - S.found_above;
  cand_round<NT>(S, cand, slots, L, lo, 11, 10, prefix, need, 1);
  prefix = (prefix << 11) | (uint32_t)S.found_bin;
  need -= S.found_above;
  cand_round<NT>(S, cand, slots, L, lo, 10, 0, prefix, need, 0);
  const uint32_t T = (prefix << 10) | (uint32_t)S.found_bin;
  const int need_eq = need - S.found_above;   // 1 <= need_eq <= the number of keys equal to T
  // every thread has read the rounds' results (cand_round ends in a barrier): reuse hist
  uint32_t* tied = &S.hist[0][0];
  for (int i = threadIdx.x; i < words; i += NT) tied[i] = 0u;
  __syncthreads();
  for_candidates<NT>(cand, slots, L, lo, [&](uint32_t key, uint32_t x) {
    if (key > T) atomicOr(&S.above[x >> 5], 1u << (x & 31));
    else if (key == T) atomicOr(&tied[x >> 5], 1u << (x & 31));
  });
  __syncthreads();
  // Ordered output.  Warp w owns words [w WPW, (w + 1) WPW) and reads them 32 at a time, lane l
  // taking word 32 r + l of round r, so the reads are conflict-free and ascending in (r, l).
  // Pass 1 counts each warp's keys > T and ties; pass 2 walks the rounds again with warp scans:
  // a tie is kept while its rank among all ties is below need_eq (the lowest indices first),
  // and every kept token's index goes to its rank among the kept ones.
  constexpr int NW = NT / 32;
  constexpr int WPW = kCandBitmapTokens / 32 / NW;   // words per warp
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wbase = warp * WPW;
  int n_above = 0, n_tied = 0;
#pragma unroll 4
  for (int r = 0; r < WPW / 32; ++r) {
    const int wi = wbase + 32 * r + lane;
    if (wi < words) {
      n_above += __popc(S.above[wi]);
      n_tied += __popc(tied[wi]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_above += __shfl_xor_sync(0xFFFFFFFFu, n_above, o);
    n_tied += __shfl_xor_sync(0xFFFFFFFFu, n_tied, o);
  }
  if (lane == 0) {
    S.scan_tmp[warp] = n_above;
    S.warp_ties[warp] = n_tied;
  }
  __syncthreads();
  int tie_run = 0, out_run = 0;   // ties and kept tokens of the warps before this one
  for (int v = 0; v < warp; ++v) {
    const int kt = min(max(need_eq - tie_run, 0), S.warp_ties[v]);
    out_run += S.scan_tmp[v] + kt;
    tie_run += S.warp_ties[v];
  }
  for (int r = 0; r < WPW / 32; ++r) {
    const int wbr = wbase + 32 * r;
    if (wbr >= words) break;   // the same in every lane of the warp
    const int wi = wbr + lane;
    const uint32_t ab = wi < words ? S.above[wi] : 0u;
    uint32_t tb = wi < words ? tied[wi] : 0u;
    // ties: this lane's rank among all ties, then how many of its own it keeps
    const int nt = __popc(tb);
    int ti = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, ti, o);
      if (lane >= o) ti += y;
    }
    const int t_rank = tie_run + ti - nt;
    int keep = min(max(need_eq - t_rank, 0), nt);
    uint32_t kept = 0u;
    while (keep-- > 0) {   // the lowest-index ties first
      const uint32_t low = tb & (0u - tb);
      kept |= low;
      tb ^= low;
    }
    uint32_t bits = ab | kept;
    const int nb = __popc(bits);
    int oi = nb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, oi, o);
      if (lane >= o) oi += y;
    }
    int pos = out_run + oi - nb;
    while (bits != 0u) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < k) out[pos] = wi * 32 + bit;
      ++pos;
    }
    out_run += __shfl_sync(0xFFFFFFFFu, oi, 31);
    tie_run += __shfl_sync(0xFFFFFFFFu, ti, 31);
  }
  for (int i = k + threadIdx.x; i < a.k_max; i += NT) out[i] = -1;
}

// The filtered scoring kernel writes no score rows.  A list the candidate path cannot serve (its
// threshold kept fewer than k scores or more than kTopkCandCap) gets its row recomputed here by
// the selection CTA -- one thread per token, an fp32 dot
// product of the bf16 query with the token's bf16 key row -- and then takes the row paths.
__device__ void rescore_row(const TopkArgs& a, int th, int b, int L, float* row, float* qs) {
  const int h = th % a.qv.hq;
  const int g = h / (a.qv.hq / a.kv.hkv);
  const uint16_t* q = static_cast<const uint16_t*>(a.qv.q) + (int64_t)th * kHeadDim;
  if (threadIdx.x < kHeadDim) qs[threadIdx.x] = __uint_as_float((uint32_t)__ldg(q + threadIdx.x) << 16);
  __syncthreads();
  for (int tok = threadIdx.x; tok < L; tok += kSelectThreads) {
    const uint32_t r = kv_row(a.kv, b, g, tok);
    float s = 0.f;
    if (r != kInvalidRow) {
      const uint4* kr = reinterpret_cast<const uint4*>(a.kv.k + (int64_t)r * kHeadDim);
#pragma unroll 4
      for (int c = 0; c < kHeadDim / 8; ++c) {
        const uint4 v = __ldg(kr + c);
        const float* qc = qs + 8 * c;
        s = fmaf(bf16lo(v.x), qc[0], s);
        s = fmaf(bf16hi(v.x), qc[1], s);
        s = fmaf(bf16lo(v.y), qc[2], s);
        s = fmaf(bf16hi(v.y), qc[3], s);
        s = fmaf(bf16lo(v.z), qc[4], s);
        s = fmaf(bf16hi(v.z), qc[5], s);
        s = fmaf(bf16lo(v.w), qc[6], s);
        s = fmaf(bf16hi(v.w), qc[7], s);
      }
    } else {
      flag_status(a.status, TSD_DEV_BAD_PAGE);
    }
    row[tok] = s;
  }
  __threadfence();   // the row paths read it back through L2
  __syncthreads();
}

// The selection over a list's score row: every visible token (k = L) or none (k = 0), the
// sampled fast path, else the multi-pass radix path.  Under the candidate filter the scoring
// kernel wrote no row, so the list's row is recomputed first.
// The same for the label indexer: the list's label scores, sum over its kv head's label channels
// of q[c] * label[row][c] in fp32, one thread per token.
__device__ void rescore_label_row(const TopkArgs& a, int th, int b, int L, float* row, float* qs) {
  const int h = th % a.qv.hq;
  const int g = h / (a.qv.hq / a.kv.hkv);
  const int R = a.label_r;
  if (threadIdx.x < R) {
    int c = __ldg(a.channels + (int64_t)g * R + threadIdx.x);
    if (c < 0 || c >= kHeadDim) c = 0;   // the scoring kernel flags it
    const int64_t qe = (int64_t)th * kHeadDim + c;
    qs[threadIdx.x] = a.qv.q_f32 ? __ldg(static_cast<const float*>(a.qv.q) + qe)
                                 : __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t*>(a.qv.q) + qe) << 16);
  }
  __syncthreads();
  for (int tok = threadIdx.x; tok < L; tok += kSelectThreads) {
    const uint32_t r = kv_row(a.kv, b, g, tok);
    float s = 0.f;
    if (r != kInvalidRow) {
      const uint16_t* lr = a.label + (int64_t)r * R;
      for (int c = 0; c < R; ++c) s = fmaf(qs[c], __uint_as_float((uint32_t)__ldg(lr + c) << 16), s);
    } else {
      flag_status(a.status, TSD_DEV_BAD_PAGE);
    }
    row[tok] = s;
  }
  __threadfence();   // the row paths read it back through L2
  __syncthreads();
}

__device__ void select_rows(SelectSmem& S, const TopkArgs& a, int th, int b, int L, int k) {
  int32_t* out = a.out_idx + (int64_t)th * a.k_max;
  float* osc = a.out_scores != nullptr ? a.out_scores + (int64_t)th * a.k_max : nullptr;
  const float* row = a.scores + (int64_t)th * a.score_stride;
  if (k == L || k == 0) {   // every visible token is kept, or none
    for (int i = threadIdx.x; i < a.k_max; i += kSelectThreads) {
      out[i] = i < k ? i : -1;
      if (osc != nullptr) osc[i] = i < k ? __ldcg(row + i) + 0.f : -CUDART_INF_F;
    }
    return;
  }
  if (a.filter) {   // the filtered scoring kernel wrote no score row: recompute this one
    __shared__ float s_q[kHeadDim];
    int L2, k2;
    if (b < 0) list_len_k(a, th, b, L2, k2);   // the list's sequence
    if (a.label != nullptr) rescore_label_row(a, th, b, L, a.scores + (int64_t)th * a.score_stride, s_q);
    else rescore_row(a, th, b, L, a.scores + (int64_t)th * a.score_stride, s_q);
  }
  if (L >= kFastMinL &&
      select_fast(S, row, a.samples + (int64_t)th * a.sample_stride, a.sample_shift, L, k, out, osc, a.k_max))
    return;
  const int tile_elems = kSelectThreads * kSelPerThread;

  // ---- pass 1: histogram of the top 11 key bits ----
  for (int i = threadIdx.x; i < kSelBins; i += kSelectThreads) S.hist[0][i] = 0u;
  __syncthreads();
  for (int base = 0; base < L; base += tile_elems) {
    const int i0 = base + threadIdx.x * kSelPerThread;
    float f[kSelPerThread];
    load16(row, i0, L, f);
#pragma unroll
    for (int j = 0; j < kSelPerThread; ++j)
      if (i0 + j < L) atomicAdd(&S.hist[0][score_key(f[j]) >> 21], 1u);
  }
  __syncthreads();
  select_bin(S, kSelBins, k);
  uint32_t prefix = (uint32_t)S.found_bin & (kSelBins - 1);
  int need = k - S.found_above;
  int ccount = (int)S.hist[0][prefix];
  int shift = 21;
  __syncthreads();

  // ---- refinement passes over global memory while the candidates do not fit ----
  while (ccount > kCandMax && shift > 0) {
    const int nb = shift >= 11 ? 11 : shift;
    shift -= nb;
    for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[0][i] = 0u;
    __syncthreads();
    for (int base = 0; base < L; base += tile_elems) {
      const int i0 = base + threadIdx.x * kSelPerThread;
      float f[kSelPerThread];
      load16(row, i0, L, f);
#pragma unroll
      for (int j = 0; j < kSelPerThread; ++j) {
        const uint32_t key = score_key(f[j]);
        if (i0 + j < L && (key >> (shift + nb)) == prefix) atomicAdd(&S.hist[0][(key >> shift) & ((1u << nb) - 1)], 1u);
      }
    }
    __syncthreads();
    select_bin(S, 1 << nb, need);
    const uint32_t d = (uint32_t)S.found_bin & ((1u << nb) - 1);
    prefix = (prefix << nb) | d;
    need -= S.found_above;
    ccount = (int)S.hist[0][d];
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
      for (int i = threadIdx.x; i < (1 << nb); i += kSelectThreads) S.hist[0][i] = 0u;
      __syncthreads();
      for (int c = threadIdx.x; c < nc; c += kSelectThreads) {
        const uint32_t key = S.cand[c];
        if ((key >> (shift + nb)) == prefix) atomicAdd(&S.hist[0][(key >> shift) & ((1u << nb) - 1)], 1u);
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

// Without the filter: one CTA per list (th = blockIdx.x).  With it (queued != 0): the lists the
// candidate kernel could not serve, taken from its queue by a grid of a few CTAs per SM; the
// last CTA to finish leaves the queue empty for the next call.
__global__ void __launch_bounds__(kSelectThreads, 2) topk_select_kernel(TopkArgs a, int queued) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelectSmem& S = *reinterpret_cast<SelectSmem*>(smem_raw);
  if (queued) {
    pdl_wait();   // the candidate kernel has queued its lists
    pdl_launch_dependents();
    const int n = (int)__ldcg(a.queue_cnt);
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
      const int th = __ldcg(a.queue + i);
      const int2 m = __ldcg(a.meta + th);
      select_rows(S, a, th, -1, m.x, m.y);
      __syncthreads();   // the next list reuses the shared memory
    }
    __shared__ int s_last;
    if (threadIdx.x == 0) s_last = atomicAdd(a.queue_done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last && threadIdx.x == 0) {
      *a.queue_cnt = 0u;
      *a.queue_done = 0u;
    }
    return;
  }
  const int th = blockIdx.x;
  int b, L, k;
  // launched as a dependent of the scoring kernel: everything before the wait reads only the
  // call's inputs; the scores are read only once that kernel has completed
  list_len_k(a, th, b, L, k);
  if (a.out_count != nullptr && threadIdx.x == 0) a.out_count[th] = k;
  pdl_wait();
  pdl_launch_dependents();
  select_rows(S, a, th, b, L, k);
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

// The filtered forms' selection (exact and label indexers): the candidate kernel, then the queue
// of lists it could not serve, each a programmatic dependent of the kernel before.
cudaError_t launch_topk_candidates(const TopkArgs& a, int num_lists, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e =
        cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SelectSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaError_t e;
  if (num_lists <= a.queue_ctas)   // at most two lists per SM: one wave of 1024-thread CTAs
    e = launch_dependent(topk_cand_kernel<1024>, dim3(num_lists), dim3(1024), 0, stream, a);
  else
    e = launch_dependent(topk_cand_kernel<256>, dim3(num_lists), dim3(256), 0, stream, a);
  if (e != cudaSuccess) return e;
  return launch_dependent(topk_select_kernel, dim3((unsigned)a.queue_ctas), dim3(kSelectThreads), sizeof(SelectSmem),
                          stream, a, 1);
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
  if (a.filter) {   // the candidate filter's pre-pass: samples and thresholds
    const dim3 g0((unsigned)a.prepass_splits, hkv * a.list_groups, batch);
    topk_prepass_kernel<<<g0, 32 * kPpWarps, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (score_on_tcgen05()) {
    if (a.qv.q_f32) {
      topk_score_tc_kernel<true><<<g1, kTcThreads, TcLayout<true>::bytes, stream>>>(a, maps);
    } else {
      topk_score_tc_kernel<false><<<g1, kTcThreads, TcLayout<false>::bytes, stream>>>(a, maps);
    }
  } else if (a.qv.q_f32) {
    topk_score_kernel<true><<<g1, kScThreads, ScLayout<true, kScStages>::bytes, stream>>>(a, maps);
  } else if (a.filter) {   // a programmatic dependent of the pre-pass: its consumers wait for lo
    cudaError_t e = launch_dependent(topk_score_kernel<false>, g1, dim3(kScThreads),
                                     (size_t)ScLayout<false, kScStages>::bytes, stream, a, maps);
    if (e != cudaSuccess) return e;
  } else {
    topk_score_kernel<false><<<g1, kScThreads, ScLayout<false, kScStages>::bytes, stream>>>(a, maps);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (!a.filter)
    return launch_dependent(topk_select_kernel, dim3(num_lists), dim3(kSelectThreads), sizeof(SelectSmem), stream, a, 0);
  return launch_topk_candidates(a, num_lists, stream);
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
  return launch_dependent(topk_select_kernel, dim3(num_lists), dim3(kSelectThreads), sizeof(SelectSmem), stream, a, 0);
}

}  // namespace tsd
