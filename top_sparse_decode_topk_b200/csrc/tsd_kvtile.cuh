// Streaming of dense K/V token tiles into shared memory and the q.K tile on tensor cores
// (shared by the dense decode and the top-k scoring kernels).
//
// A tile is 64 consecutive tokens of one (sequence, kv head).  Each 256-byte row is
// stored as two 128-byte halves (dims 0-63, 64-127), each half a [64 rows][128 B] block
// written with 128-byte swizzling (16-byte chunk index XOR row mod 8), so that ldmatrix
// reads of 8 rows hit 8 different bank groups.  The tile arrives through TMA 2-D loads of
// 16-token (or page-sized, >= 8) boxes -- one load per box and per half -- counted on the
// stage's "full" mbarrier; caches with pages smaller than 8 tokens fall back to 16-byte
// cp.async copies into the same swizzled layout, signalled through the same barrier.
//
// Tensor-core math is the warp-level bf16 mma.m16n8k16 with fp32 accumulation: the 16
// query vectors of a CTA (q heads of the GQA group x decode tokens) are the M dimension,
// 8 tokens the N dimension, 16 head dims the K dimension.  Products of bf16 values are
// exact in fp32; fp32 queries are split into bf16 hi + lo parts (two MMAs).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tsd_common.cuh"

namespace tsd {

constexpr int kTileTok = 64;
constexpr int kHalfBytes = kTileTok * 128;   // one 128-byte half of a 64-row tile
constexpr int kTileBytesKV = 2 * kHalfBytes;  // one tensor (K or V) of a tile: 16 KB

struct KvMaps {
  CUtensorMap k;   // [rows][128] bf16, box {64, box_rows}, 128-byte swizzle
  CUtensorMap v;
};

// Box rows of the TMA tensor maps: 16-token boxes, or one page when pages are 8 tokens.
__device__ __forceinline__ int tma_box_rows(const KvView& kv) {
  return kv.page_table == nullptr ? 16 : min(16, 1 << kv.page_shift);
}

// Row coordinate (in the [rows][128] view) of the box that starts at token t of (b, g):
// -1 past tok_end, -2 for a bad page (flagged).
__device__ __forceinline__ int tma_box_y(const KvView& kv, int b, int g, int t, int tok_end, uint32_t* status) {
  if (t >= tok_end) return -1;
  if (kv.page_table == nullptr) return (b * kv.hkv + g) * kv.max_seq_len + t;
  const int32_t page = __ldg(kv.page_table + (int64_t)b * kv.max_pages + (t >> kv.page_shift));
  if (page < 0 || (int64_t)page >= kv.num_pages) {
    flag_status(status, TSD_DEV_BAD_PAGE);
    return -2;
  }
  return (int)((((int64_t)page * kv.hkv + g) << kv.page_shift) | (t & ((1 << kv.page_shift) - 1)));
}

// Producer-warp view of the box coordinates of a window: lane i holds the coordinate of box
// 32 s + i of the current segment s and prefetches segment s + 1, so page-table lookups
// cost one round trip per 32 boxes and are off the issue path.
struct BoxRows {
  int cur, nxt, seg;
};

__device__ __forceinline__ void box_rows_init(BoxRows& br, const KvView& kv, int b, int g, int tok0, int tok_end,
                                              int bp, int lane, uint32_t* status) {
  br.seg = 0;
  br.cur = tma_box_y(kv, b, g, tok0 + lane * bp, tok_end, status);
  br.nxt = tma_box_y(kv, b, g, tok0 + (32 + lane) * bp, tok_end, status);
}

// Coordinate of box `box` of the window; all 32 lanes must call it with the same box.
__device__ __forceinline__ int box_rows_get(BoxRows& br, const KvView& kv, int b, int g, int tok0, int tok_end, int bp,
                                            int lane, int box, uint32_t* status) {
  const int seg = box >> 5;
  while (br.seg < seg) {
    br.cur = br.nxt;
    ++br.seg;
    br.nxt = tma_box_y(kv, b, g, tok0 + ((br.seg + 1) * 32 + lane) * bp, tok_end, status);
  }
  return __shfl_sync(0xFFFFFFFFu, br.cur, box & 31);
}

// Issue the TMA loads of one TT-token tile (all 32 lanes call it; lane 0 issues) and
// return the bytes issued (valid on lane 0).  Each K/V half is a [TT rows][128 B] block.
template <int TT = kTileTok>
__device__ __forceinline__ uint32_t tile_issue_tma(const KvView& kv, const CUtensorMap* tmk, const CUtensorMap* tmv,
                                                   BoxRows& br, int b, int g, int tok0, int tok_end, int tile,
                                                   unsigned char* kdst, unsigned char* vdst, uint64_t* bar, int lane,
                                                   uint32_t* status) {
  const int bp = tma_box_rows(kv);
  uint32_t bytes = 0;
  for (int r = 0; r < TT; r += bp) {
    const int box = (tile * TT + r) / bp;
    const int y = box_rows_get(br, kv, b, g, tok0, tok_end, bp, lane, box, status);
    if (y == -1) break;
    if (y < 0) continue;
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();
      tma_load_2d_hint(kdst + r * 128, tmk, 0, y, bar, pol);
      tma_load_2d_hint(kdst + TT * 128 + r * 128, tmk, 64, y, bar, pol);
      if (vdst != nullptr) {
        tma_load_2d_hint(vdst + r * 128, tmv, 0, y, bar, pol);
        tma_load_2d_hint(vdst + TT * 128 + r * 128, tmv, 64, y, bar, pol);
      }
    }
    bytes += (vdst != nullptr ? 4 : 2) * bp * 128;
  }
  return bytes;
}

// cp.async path (pages < 8 tokens): called by all 32 lanes of the producer warp.
template <int TT = kTileTok>
__device__ __forceinline__ void tile_issue_cpasync(const KvView& kv, int b, int g, int tok, int tok_end,
                                                   unsigned char* kdst, unsigned char* vdst, int lane,
                                                   uint32_t* status) {
  const int ntensor = vdst != nullptr ? 2 : 1;
  // TT rows x 16 chunks per tensor; lane -> (row, chunk) pairs
  for (int id = lane; id < TT * 16 * ntensor; id += 32) {
    const int which = id / (TT * 16);
    const int rc = id % (TT * 16);
    const int r = rc >> 4, ch = rc & 15;
    const int t = tok + r;
    if (t >= tok_end) continue;
    const uint32_t row = kv_row(kv, b, g, t);
    if (row == kInvalidRow) {
      if (ch == 0) flag_status(status, TSD_DEV_BAD_PAGE);
      continue;
    }
    const uint16_t* src = (which ? kv.v : kv.k) + (int64_t)row * kHeadDim + ch * 8;
    unsigned char* base = which ? vdst : kdst;
    cp_async16_hint(base + (ch >> 3) * (TT * 128) + sw128(r, ch & 7), src, l2_evict_first());
  }
}

__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Producer warp of a tile ring (all 32 lanes call it).  Streams tiles [0, ntiles) of the
// window [tok0, tok_end) of (sequence b, kv head g) into stage tile % NST: K at the start of
// the stage and, WITH_V, V kTileBytesKV after it.  `full[s]` counts the bytes of a fill
// (TMA) or the 32 lanes' copies (cp.async); `empty[s]` the consumer warps' releases.  Every
// wait is bounded: on a timeout the producer flags TSD_DEV_TIMEOUT, raises `abort` and
// stops.  Before returning it waits for its last fills to land, so that no copy into shared
// memory is in flight when the CTA ends.
template <int NST, int STAGE_BYTES, bool WITH_V, int TT = kTileTok>
__device__ __forceinline__ void produce_tiles(const KvView& kv, const KvMaps& maps, int b, int g, int tok0,
                                              int tok_end, int ntiles, unsigned char* stages, uint64_t* full,
                                              uint64_t* empty, uint32_t* abort, bool use_tma, int lane,
                                              uint32_t* status) {
  constexpr uint32_t kLoadsPerBox = WITH_V ? 4 : 2;
  BoxRows br;
  const int bp = tma_box_rows(kv);
  if (use_tma) box_rows_init(br, kv, b, g, tok0, tok_end, bp, lane, status);
  int issued = 0;
  for (int tile = 0; tile < ntiles; ++tile) {
    const int s = tile % NST;
    if (tile >= NST) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[s], ((tile / NST) - 1) & 1);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          flag_status(status, TSD_DEV_TIMEOUT);
          atomicOr(abort, 1u);
        }
        break;
      }
    }
    unsigned char* kd = stages + (size_t)s * STAGE_BYTES;
    unsigned char* vd = WITH_V ? kd + 2 * TT * 128 : nullptr;
    const int tok = tok0 + tile * TT;
    if (use_tma) {
      // the expected bytes must be registered before the loads can complete the phase
      const int rows = min(TT, tok_end - tok);
      const uint32_t want = (uint32_t)((rows + bp - 1) / bp) * kLoadsPerBox * bp * 128;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], want);
      __syncwarp();
      const uint32_t got = tile_issue_tma<TT>(kv, &maps.k, &maps.v, br, b, g, tok0, tok_end, tile, kd, vd, &full[s],
                                              lane, status);
      // boxes skipped for a bad page never arrive: complete their bytes so the phase ends
      if (lane == 0 && got < want) mbar_complete_tx(&full[s], want - got);
    } else {
      tile_issue_cpasync<TT>(kv, b, g, tok, tok_end, kd, vd, lane, status);
      cp_async_mbar_arrive(&full[s]);
    }
    issued = tile + 1;
  }
  if (lane == 0) {
    for (int tile = (issued > NST ? issued - NST : 0); tile < issued; ++tile)
      if (!mbar_wait(&full[tile % NST], (tile / NST) & 1)) flag_status(status, TSD_DEV_TIMEOUT);
  }
}

// Consumer warp: wait (bounded) for tile `tile` of the ring.  False on a timeout (flagged)
// or when the producer has given up.
template <int NST>
__device__ __forceinline__ bool consume_wait(uint64_t* full, const uint32_t* abort, int tile, int lane,
                                             uint32_t* status) {
  bool ok = true;
  if (lane == 0) ok = mbar_wait(&full[tile % NST], (tile / NST) & 1);
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (!ok && lane == 0) flag_status(status, TSD_DEV_TIMEOUT);
  return ok && *reinterpret_cast<const volatile uint32_t*>(abort) == 0u;
}

// Query tile (mma A operand, 16 rows x 128 dims) in shared memory, laid out like a K tile
// (two 128-byte halves of [16 rows][128 B], 128-byte swizzled): row m is list m of the CTA
// (token j = m / G of the sequence, q head g * G + m % G); rows >= nlists are zero.  For
// fp32 queries a second tile holds the bf16 remainders q - bf16(q).
constexpr int kQHalfBytes = 16 * 128;
constexpr int kQTileBytes = 2 * kQHalfBytes;

// Called by `nthreads` threads (index tid): fills qhi (and qlo when non-null).
__device__ __forceinline__ void store_q_tile(const QView& qv, const SeqInfo& si, int g, int G, int m0, int nlists,
                                             unsigned char* qhi, unsigned char* qlo, int tid, int nthreads) {
  for (int i = tid; i < 16 * 16; i += nthreads) {   // 16 rows x 16 chunks of 8 dims
    const int m = i >> 4, ch = i & 15;
    uint4 hi = make_uint4(0, 0, 0, 0), lo = make_uint4(0, 0, 0, 0);
    if (m < nlists) {
      const int mg = m0 + m;
      const int j = mg / G;
      const int64_t base = ((int64_t)(si.t0 + j) * qv.hq + g * G + (mg - j * G)) * kHeadDim + ch * 8;
      if (qv.q_f32) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(qv.q) + base));
        const float4 y = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(qv.q) + base + 4));
        split_bf16(x.x, x.y, hi.x, lo.x);
        split_bf16(x.z, x.w, hi.y, lo.y);
        split_bf16(y.x, y.y, hi.z, lo.z);
        split_bf16(y.z, y.w, hi.w, lo.w);
      } else {
        hi = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(qv.q) + base));
      }
    }
    const uint32_t off = (ch >> 3) * kQHalfBytes + sw128(m, ch & 7);
    *reinterpret_cast<uint4*>(qhi + off) = hi;
    if (qlo != nullptr) *reinterpret_cast<uint4*>(qlo + off) = lo;
  }
}

// A fragment of k-step ks from a query tile.
__device__ __forceinline__ void q_frag(const unsigned char* qt, int ks, int lane, uint32_t* a) {
  const int i4 = lane >> 3;
  const int row = ((i4 & 1) << 3) + (lane & 7);
  const int chunk = ((ks & 3) << 1) + (i4 >> 1);
  ldsm_x4(smem_u32(qt) + (ks >> 2) * kQHalfBytes + sw128(row, chunk), a[0], a[1], a[2], a[3]);
}

// S(16 queries x 16 tokens) of one warp: tokens [16 w, 16 w + 16) of the tile in stage K.
// S[nt][0..1] = (query lane/4, tokens 8 nt + 2 (lane%4) + {0,1}); S[nt][2..3] = query lane/4 + 8.
// With SPLIT the even and odd k-steps accumulate separately and are added at the end, which
// halves the chain of dependent MMAs (the scores then round in that order).
template <bool QF32, bool SPLIT = false>
__device__ __forceinline__ void qk_tile(const unsigned char* qhi, const unsigned char* qlo, const unsigned char* ktile,
                                        int w, int lane, float S[2][4]) {
  float T[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      S[nt][i] = 0.f;
      T[nt][i] = 0.f;
    }
  const int i4 = lane >> 3, rr = lane & 7;
  const int tokrow = 16 * w + ((i4 >> 1) << 3) + rr;
  const uint32_t kbase = smem_u32(ktile);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int chunk = ((ks & 3) << 1) + (i4 & 1);
    uint32_t b00, b01, b10, b11;
    ldsm_x4(kbase + (ks >> 2) * kHalfBytes + sw128(tokrow, chunk), b00, b01, b10, b11);
    uint32_t a[4];
    q_frag(qhi, ks, lane, a);
    float (*D)[4] = (SPLIT && (ks & 1)) ? T : S;
    mma_bf16(D[0], a, b00, b01);
    mma_bf16(D[1], a, b10, b11);
    if (QF32) {
      q_frag(qlo, ks, lane, a);
      mma_bf16(D[0], a, b00, b01);
      mma_bf16(D[1], a, b10, b11);
    }
  }
  if (SPLIT) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) S[nt][i] += T[nt][i];
  }
}

}  // namespace tsd
