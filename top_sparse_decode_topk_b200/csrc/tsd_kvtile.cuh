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

// Load the tokens [tok, min(tok + 64, tok_end)) of (b, g) into one stage.
// K goes to kdst (16 KB, 1024-byte aligned), V to vdst (or nothing when vdst is null).
// TMA path: called by one lane; returns the bytes the stage's barrier must expect.
__device__ __forceinline__ uint32_t tile_issue_tma(const KvView& kv, const CUtensorMap* tmk, const CUtensorMap* tmv,
                                                   int b, int g, int tok, int tok_end, unsigned char* kdst,
                                                   unsigned char* vdst, uint64_t* bar, uint32_t* status) {
  const int bp = kv.page_table == nullptr ? 16 : min(16, 1 << kv.page_shift);   // box rows
  uint32_t bytes = 0;
  for (int r = 0; r < kTileTok; r += bp) {
    const int t = tok + r;
    if (t >= tok_end) break;
    int y;
    if (kv.page_table == nullptr) {
      y = (b * kv.hkv + g) * kv.max_seq_len + t;
    } else {
      const int32_t page = __ldg(kv.page_table + (int64_t)b * kv.max_pages + (t >> kv.page_shift));
      if (page < 0 || (int64_t)page >= kv.num_pages) {
        flag_status(status, TSD_DEV_BAD_PAGE);
        continue;
      }
      y = (int)((((int64_t)page * kv.hkv + g) << kv.page_shift) | (t & ((1 << kv.page_shift) - 1)));
    }
    tma_load_2d(kdst + r * 128, tmk, 0, y, bar);
    tma_load_2d(kdst + kHalfBytes + r * 128, tmk, 64, y, bar);
    bytes += 2 * bp * 128;
    if (vdst != nullptr) {
      tma_load_2d(vdst + r * 128, tmv, 0, y, bar);
      tma_load_2d(vdst + kHalfBytes + r * 128, tmv, 64, y, bar);
      bytes += 2 * bp * 128;
    }
  }
  return bytes;
}

// cp.async path (pages < 8 tokens): called by all 32 lanes of the producer warp.
__device__ __forceinline__ void tile_issue_cpasync(const KvView& kv, int b, int g, int tok, int tok_end,
                                                   unsigned char* kdst, unsigned char* vdst, int lane,
                                                   uint32_t* status) {
  const int ntensor = vdst != nullptr ? 2 : 1;
  // 64 rows x 16 chunks per tensor; lane -> (row, chunk) pairs
  for (int id = lane; id < kTileTok * 16 * ntensor; id += 32) {
    const int which = id / (kTileTok * 16);
    const int rc = id % (kTileTok * 16);
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
    cp_async16(base + (ch >> 3) * kHalfBytes + sw128(r, ch & 7), src);
  }
}

// Query fragments (mma A operand, 16 rows x 128 dims): row m is list m of the CTA (token
// j = m / G of the sequence, q head g * G + m % G); rows >= nlists are zero.  For fp32
// queries the lo parts carry q - bf16(q).
template <bool QF32>
struct QFrags {
  uint32_t hi[8][4];
  uint32_t lo[QF32 ? 8 : 1][4];
};

template <bool QF32>
__device__ __forceinline__ void load_q_frags(const QView& qv, const SeqInfo& si, int g, int G, int m0, int nlists,
                                             int lane, QFrags<QF32>& f) {
  const int r0 = lane >> 2, kk = (lane & 3) * 2;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int m = r0 + 8 * half;
    const bool ok = m < nlists;
    const int mg = m0 + m;
    const int j = mg / G;
    const int64_t base = ((int64_t)(si.t0 + j) * qv.hq + g * G + (mg - j * G)) * kHeadDim;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int hk = 0; hk < 2; ++hk) {
        const int d = ks * 16 + kk + 8 * hk;
        uint32_t hi = 0, lo = 0;
        if (ok) {
          if (QF32) {
            const float2 x = __ldg(reinterpret_cast<const float2*>(reinterpret_cast<const float*>(qv.q) + base + d));
            split_bf16(x.x, x.y, hi, lo);
          } else {
            hi = __ldg(reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(qv.q) + base + d));
          }
        }
        // a0 = (row r0, k lo), a1 = (row r0 + 8, k lo), a2 = (row r0, k hi), a3 = (row r0 + 8, k hi)
        f.hi[ks][half + 2 * hk] = hi;
        if (QF32) f.lo[ks][half + 2 * hk] = lo;
      }
    }
  }
}

// S(16 queries x 16 tokens) of one warp: tokens [16 w, 16 w + 16) of the tile in stage K.
// S[nt][0..1] = (query lane/4, tokens 8 nt + 2 (lane%4) + {0,1}); S[nt][2..3] = query lane/4 + 8.
template <bool QF32>
__device__ __forceinline__ void qk_tile(const QFrags<QF32>& f, const unsigned char* ktile, int w, int lane,
                                        float S[2][4]) {
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) S[nt][i] = 0.f;
  const int i4 = lane >> 3, rr = lane & 7;
  const int tokrow = 16 * w + ((i4 >> 1) << 3) + rr;
  const uint32_t kbase = smem_u32(ktile);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int chunk = ((ks & 3) << 1) + (i4 & 1);
    uint32_t b00, b01, b10, b11;
    ldsm_x4(kbase + (ks >> 2) * kHalfBytes + sw128(tokrow, chunk), b00, b01, b10, b11);
    mma_bf16(S[0], f.hi[ks], b00, b01);
    mma_bf16(S[1], f.hi[ks], b10, b11);
    if (QF32) {
      mma_bf16(S[0], f.lo[ks], b00, b01);
      mma_bf16(S[1], f.lo[ks], b10, b11);
    }
  }
}

}  // namespace tsd
