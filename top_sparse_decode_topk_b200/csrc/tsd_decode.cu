// Sparse and dense decode attention kernels for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?",
// gist.science summary, section 2 "Hardware implementation" and section 3.C):
// for each (query token t, q head h) attend only to the K/V rows named by its
// index list -- which may differ per token, per query and per head -- so that
// the bytes read fall from O(N d) to O(k d).  Dense decode attends to every row.
//
// Work unit (one CTA): sequence b, kv head g, a group of up to 32 query lists
// (q heads of the GQA group x decode tokens of the sequence) and one split of
// the work: a chunk of E consecutive entries of every list (sparse) or a window
// of W consecutive tokens (dense).
//
// Sparse CTA, in order:
//   1. load the chunk's entries of every list, validate and compact them;
//   2. deduplicate the rows across lists with a bitmap over the chunk's token
//      span (one bit per token; a prefix popcount gives each row its slot), so
//      a row picked by several heads or tokens is loaded once;
//   3. stream the unique rows through a 4-stage cp.async ring of 16-row tiles
//      (16-byte copies; K and V rows are 256 bytes each);
//   4. 32 lane-groups of 8 lanes walk the lists: each entry's score is a 16-wide
//      fp32 dot per lane reduced over the group with 3 shuffles, followed by an
//      online-softmax update of the group's (max, sum, 128-wide row) state;
//   5. combine the groups of a list, write the split's partial, and the last
//      CTA of the (b, g, list group) to arrive merges the splits (log-sum-exp).
// No CTA ever waits on another: the merge is done by whichever arrives last.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"

namespace tsd {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kTileBytes = kRowsPerTile * 2 * 256;          // K rows then V rows
constexpr int kRingBytes = kStages * kTileBytes;
constexpr int kCombFloats = 132;                             // m, l, pad, pad, acc[128]
constexpr int kMaxTiles = kMaxEntriesPerCta / kRowsPerTile;  // tiles per sparse CTA


// List m of a CTA -> (token, q head).  Lists are ordered token-major inside a sequence:
// global list j*G + hh is token j (of the sequence) and q head g*G + hh.
struct ListRef {
  int t;      // query token, -1 if the list does not exist
  int h;
  int kvlen;
};

__device__ __forceinline__ ListRef list_ref(const DecodeArgs& a, const SeqInfo& si, int g, int lg, int m) {
  ListRef r;
  const int G = a.qv.hq / a.kv.hkv;
  const int mg = lg * a.lists_per_cta + m;
  if (m >= a.lists_per_cta || mg >= si.n * G) {
    r.t = -1; r.h = 0; r.kvlen = 0;
    return r;
  }
  const int j = mg / G;
  r.t = si.t0 + j;
  r.h = g * G + (mg - j * G);
  r.kvlen = kv_len_of(a.qv, si, j);
  return r;
}

// Load 16 query values of list (t, h) owned by lane `l8` of a group: dims
// [8*l8, 8*l8+8) and [64+8*l8, 64+8*l8+8), pre-multiplied by scale*log2(e) so that
// dot products come out in base-2 softmax units.
__device__ __forceinline__ void load_q16(const QView& qv, int t, int h, int l8, float scale, float* q) {
  const int64_t base = ((int64_t)t * qv.hq + h) * kHeadDim;
  if (qv.q_f32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(qv.q) + base);
    float4 a0 = __ldg(p + 2 * l8), a1 = __ldg(p + 2 * l8 + 1);
    float4 b0 = __ldg(p + 16 + 2 * l8), b1 = __ldg(p + 16 + 2 * l8 + 1);
    float v[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                   b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = v[j] * scale;
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(qv.q) + base);
    uint4 a0 = __ldg(p + l8), b0 = __ldg(p + 8 + l8);
    float v[16];
    unpack8(a0, v);
    unpack8(b0, v + 8);
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = v[j] * scale;
  }
}

// Dot of a 256-byte bf16 row in shared memory with the lane's 16 query values,
// summed over the 8 lanes of the group (full-warp shuffles: call warp-uniformly).
__device__ __forceinline__ float group_dot(const unsigned char* row, int l8, const float* q) {
  uint4 k0 = *reinterpret_cast<const uint4*>(row + 16 * l8);
  uint4 k1 = *reinterpret_cast<const uint4*>(row + 128 + 16 * l8);
  float kf[16];
  unpack8(k0, kf);
  unpack8(k1, kf + 8);
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s0 = fmaf(q[j], kf[j], s0);
    s1 = fmaf(q[8 + j], kf[8 + j], s1);
  }
  float s = s0 + s1;
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 4);
  return s;
}

// Online-softmax state of one lane-group for one list.
struct SoftState {
  float m, l;
  float acc[16];
};

__device__ __forceinline__ void soft_init(SoftState& st) {
  st.m = -CUDART_INF_F;
  st.l = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) st.acc[j] = 0.f;
}

__device__ __forceinline__ void soft_update(SoftState& st, float s, const unsigned char* vrow, int l8) {
  if (s > st.m) {
    const float alpha = fast_exp2(st.m - s);
    st.l *= alpha;
#pragma unroll
    for (int j = 0; j < 16; ++j) st.acc[j] *= alpha;
    st.m = s;
  }
  const float p = fast_exp2(s - st.m);
  st.l += p;
  uint4 v0 = *reinterpret_cast<const uint4*>(vrow + 16 * l8);
  uint4 v1 = *reinterpret_cast<const uint4*>(vrow + 128 + 16 * l8);
  float vf[16];
  unpack8(v0, vf);
  unpack8(v1, vf + 8);
#pragma unroll
  for (int j = 0; j < 16; ++j) st.acc[j] = fmaf(p, vf[j], st.acc[j]);
}

// Write a group's state into the combine buffer entry `slot` (lane l8 owns 16 dims).
__device__ __forceinline__ void soft_store(float* comb, int slot, const SoftState& st, int l8) {
  float* e = comb + (size_t)slot * kCombFloats;
  if (l8 == 0) {
    e[0] = st.m;
    e[1] = st.l;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    e[4 + 8 * l8 + j] = st.acc[j];
    e[4 + 64 + 8 * l8 + j] = st.acc[8 + j];
  }
}

__device__ __forceinline__ void store_out(const DecodeArgs& a, int t, int h, int d, float v) {
  const int64_t o = ((int64_t)t * a.qv.hq + h) * kHeadDim + d;
  if (a.out_f32) {
    reinterpret_cast<float*>(a.out)[o] = v;
  } else {
    reinterpret_cast<uint16_t*>(a.out)[o] = f32_to_bf16_rne(v);
  }
}

// Combine the `nparts` states of each of the CTA's lists held in `comb`
// (entry list*nparts + part), then either write the final rows (single split) or
// this split's partial, count the arrival, and -- if this CTA is the last of its
// (b, g, list group) -- merge all splits.
__device__ void finish_lists(const DecodeArgs& a, const SeqInfo& si, int b, int g, int lg, int split,
                             int nlists, int nparts, const float* comb, float* sm_mx, float* sm_l) {
  // 1. per-list combine over parts
  for (int i = threadIdx.x; i < nlists * kHeadDim; i += blockDim.x) {
    const int m = i / kHeadDim, d = i % kHeadDim;
    const ListRef r = list_ref(a, si, g, lg, m);
    if (r.t < 0) continue;
    float mx = -CUDART_INF_F;
    for (int p = 0; p < nparts; ++p) mx = fmaxf(mx, comb[(size_t)(m * nparts + p) * kCombFloats]);
    float L = 0.f, A = 0.f;
    if (mx != -CUDART_INF_F) {
      for (int p = 0; p < nparts; ++p) {
        const float* e = comb + (size_t)(m * nparts + p) * kCombFloats;
        const float w = fast_exp2(e[0] - mx);
        L = fmaf(w, e[1], L);
        A = fmaf(w, e[4 + d], A);
      }
    }
    if (a.nsplit == 1) {
      store_out(a, r.t, r.h, d, L > 0.f ? A / L : 0.f);
      if (d == 0 && a.lse != nullptr)
        a.lse[(int64_t)r.t * a.qv.hq + r.h] = L > 0.f ? (mx + log2f(L)) * kLn2 : -CUDART_INF_F;
    } else {
      const int64_t pidx = ((int64_t)r.t * a.qv.hq + r.h) * a.nsplit + split;
      a.part_acc[pidx * kHeadDim + d] = A;
      if (d == 0) a.part_ml[pidx] = make_float2(mx, L);
    }
  }
  if (a.nsplit == 1) return;

  // 2. arrival count; the last CTA of the unit merges
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t* ctr = a.counters + ((int64_t)b * a.kv.hkv + g) * a.list_groups + lg;
    const uint32_t prev = atomicAdd(ctr, 1u);
    s_last = (prev == (uint32_t)(a.nsplit - 1));
    if (s_last) atomicExch(ctr, 0u);   // leave the counter zero for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // 3. merge the splits of every list: max and sum per list, then the rows
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int m = warp; m < nlists; m += blockDim.x / 32) {
    const ListRef r = list_ref(a, si, g, lg, m);
    if (r.t < 0) continue;
    const float2* ml = a.part_ml + ((int64_t)r.t * a.qv.hq + r.h) * a.nsplit;
    float mx = -CUDART_INF_F;
    for (int c = lane; c < a.nsplit; c += 32) mx = fmaxf(mx, __ldcg(&ml[c]).x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    float L = 0.f;
    if (mx != -CUDART_INF_F)
      for (int c = lane; c < a.nsplit; c += 32) {
        const float2 v = __ldcg(&ml[c]);
        L = fmaf(fast_exp2(v.x - mx), v.y, L);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
    if (lane == 0) {
      sm_mx[m] = mx;
      sm_l[m] = L;
      if (a.lse != nullptr)
        a.lse[(int64_t)r.t * a.qv.hq + r.h] = L > 0.f ? (mx + log2f(L)) * kLn2 : -CUDART_INF_F;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nlists * kHeadDim; i += blockDim.x) {
    const int m = i / kHeadDim, d = i % kHeadDim;
    const ListRef r = list_ref(a, si, g, lg, m);
    if (r.t < 0) continue;
    const float mx = sm_mx[m], L = sm_l[m];
    float A = 0.f;
    if (L > 0.f) {
      const int64_t pbase = ((int64_t)r.t * a.qv.hq + r.h) * a.nsplit;
      for (int c = 0; c < a.nsplit; ++c) {
        const float w = fast_exp2(__ldcg(&a.part_ml[pbase + c]).x - mx);
        if (w > 0.f) A = fmaf(w, __ldcg(&a.part_acc[(pbase + c) * kHeadDim + d]), A);
      }
    }
    store_out(a, r.t, r.h, d, L > 0.f ? A / L : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Sparse decode
// ---------------------------------------------------------------------------
struct SparseSmem {
  unsigned char ring[kRingBytes];              // also the combine buffer at the end
  uint32_t ent_tok[kMaxEntriesPerCta];         // compacted entries, list m at m*E
  uint16_t ent_slot[kMaxEntriesPerCta];        // unique-row slot of each entry
  uint32_t rowaddr[kMaxEntriesPerCta];         // physical row of each slot
  uint32_t bitmap[kBitmapWords];
  int wbase[kBitmapWords];
  uint16_t bnd[kMaxListsPerCta][kMaxTiles + 1];  // first entry of each tile, per list
  int list_n[kMaxListsPerCta];
  int list_off[kMaxListsPerCta + 1];
  int scan_tmp[kDecodeThreads / 32 + 1];
  int tmin, tmax, nunique;
  float mx[kMaxListsPerCta], lsum[kMaxListsPerCta];
};
static_assert(kStages * kTileBytes >= kMaxListsPerCta * kCombFloats * 4, "combine buffer must fit the ring");

__device__ __forceinline__ void load_tile(SparseSmem& S, const KvView& kv, int tile, int nunique) {
  const int stage = tile % kStages;
  unsigned char* base = S.ring + stage * kTileBytes;
#pragma unroll
  for (int q = 0; q < (kRowsPerTile * 32) / kDecodeThreads; ++q) {
    const int id = threadIdx.x + q * kDecodeThreads;
    const int r = id >> 5, which = (id >> 4) & 1, ch = id & 15;
    const int slot = tile * kRowsPerTile + r;
    if (slot < nunique) {
      const uint32_t row = S.rowaddr[slot];
      if (row != kInvalidRow) {
        const uint16_t* src = (which ? kv.v : kv.k) + (int64_t)row * kHeadDim + ch * 8;
        cp_async16(base + which * (kRowsPerTile * 256) + r * 256 + ch * 16, src);
      }
    }
  }
}

__global__ void __launch_bounds__(kDecodeThreads, 2) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SparseSmem& S = *reinterpret_cast<SparseSmem*>(smem_raw);

  const int split = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.span;

  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, split == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;   // uniform over the whole (b, g, lg) unit: no merge is owed

  // ---- 1. entries: load, validate, compact (warp per list) ----
  for (int m = warp; m < nlists; m += kDecodeThreads / 32) {
    const ListRef r = list_ref(a, si, g, lg, m);
    const int32_t* lst = a.idx + ((int64_t)r.t * a.qv.hq + r.h) * a.k_max;
    const int e0 = split * E;
    int e1 = e0 + E;
    if (e1 > a.k_max) e1 = a.k_max;
    uint32_t prev = (e0 > 0) ? (uint32_t)__ldg(lst + e0 - 1) : 0u;
    int count = 0;
    uint32_t bad = 0;
    for (int base = e0; base < e1; base += 32) {
      const int e = base + lane;
      const int32_t v = e < e1 ? __ldg(lst + e) : -1;
      uint32_t before = __shfl_up_sync(0xFFFFFFFFu, (uint32_t)v, 1);
      if (lane == 0) before = prev;
      if (e < e1 && (e > 0) && (uint32_t)v < before) bad |= TSD_DEV_UNSORTED;
      if (e < e1 && (v < -1 || v >= r.kvlen)) bad |= TSD_DEV_BAD_INDEX;
      const bool ok = e < e1 && v >= 0 && v < r.kvlen;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, ok);
      if (ok) S.ent_tok[m * E + count + __popc(bal & ((1u << lane) - 1))] = (uint32_t)v;
      count += __popc(bal);
      prev = __shfl_sync(0xFFFFFFFFu, (uint32_t)v, 31);
    }
    bad = __reduce_or_sync(0xFFFFFFFFu, bad);
    if (lane == 0) {
      S.list_n[m] = count;
      if (bad) flag_status(a.status, bad);
    }
  }
  if (threadIdx.x == 0) {
    S.tmin = 0x7FFFFFFF;
    S.tmax = -1;
  }
  __syncthreads();

  // ---- 2. token span of the chunk ----
  {
    int lo = 0x7FFFFFFF, hi = -1;
    for (int m = 0; m < nlists; ++m) {
      const int n = S.list_n[m];
      for (int e = threadIdx.x; e < n; e += kDecodeThreads) {
        const int v = (int)S.ent_tok[m * E + e];
        lo = min(lo, v);
        hi = max(hi, v);
      }
    }
    lo = __reduce_min_sync(0xFFFFFFFFu, lo);
    hi = __reduce_max_sync(0xFFFFFFFFu, hi);
    if (lane == 0) {
      atomicMin(&S.tmin, lo);
      atomicMax(&S.tmax, hi);
    }
  }
  if (threadIdx.x == 0) {
    int off = 0;
    for (int m = 0; m < nlists; ++m) {
      S.list_off[m] = off;
      off += S.list_n[m];
    }
    S.list_off[nlists] = off;
  }
  __syncthreads();

  // ---- 3. deduplicate rows: bitmap over the span, prefix popcount -> slots ----
  const int tmin = S.tmin;
  const int span = S.tmax - tmin + 1;
  int nunique;
  if (S.tmax >= 0 && span <= kBitmapWords * 32) {
    const int nwords = (span + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += kDecodeThreads) S.bitmap[w] = 0u;
    __syncthreads();
    for (int m = 0; m < nlists; ++m) {
      const int n = S.list_n[m];
      for (int e = threadIdx.x; e < n; e += kDecodeThreads) {
        const int o = (int)S.ent_tok[m * E + e] - tmin;
        atomicOr(&S.bitmap[o >> 5], 1u << (o & 31));
      }
    }
    __syncthreads();
    constexpr int kWordsPerThread = kBitmapWords / kDecodeThreads;
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kWordsPerThread; ++j) {
      const int w = threadIdx.x * kWordsPerThread + j;
      cnt += (w < nwords) ? __popc(S.bitmap[w]) : 0;
    }
    int total;
    int run = block_exclusive_scan<kDecodeThreads>(cnt, S.scan_tmp, &total);
#pragma unroll
    for (int j = 0; j < kWordsPerThread; ++j) {
      const int w = threadIdx.x * kWordsPerThread + j;
      if (w < nwords) {
        S.wbase[w] = run;
        // physical rows of the unique tokens, in token order
        uint32_t bits = S.bitmap[w];
        int slot = run;
        while (bits) {
          const int bit = __ffs(bits) - 1;
          bits &= bits - 1;
          const int tok = tmin + w * 32 + bit;
          const uint32_t row = kv_row(a.kv, b, g, tok);
          if (row == kInvalidRow) flag_status(a.status, TSD_DEV_BAD_PAGE);
          S.rowaddr[slot++] = row;
        }
        run += __popc(S.bitmap[w]);
      }
    }
    nunique = total;
    __syncthreads();
    for (int m = 0; m < nlists; ++m) {
      const int n = S.list_n[m];
      for (int e = threadIdx.x; e < n; e += kDecodeThreads) {
        const int o = (int)S.ent_tok[m * E + e] - tmin;
        const uint32_t word = S.bitmap[o >> 5];
        S.ent_slot[m * E + e] = (uint16_t)(S.wbase[o >> 5] + __popc(word & ((1u << (o & 31)) - 1u)));
      }
    }
  } else {
    // span too wide for the bitmap: every entry is its own row (no dedupe)
    nunique = S.list_off[nlists];
    for (int m = 0; m < nlists; ++m) {
      const int n = S.list_n[m];
      for (int e = threadIdx.x; e < n; e += kDecodeThreads) {
        const int slot = S.list_off[m] + e;
        const uint32_t row = kv_row(a.kv, b, g, (int)S.ent_tok[m * E + e]);
        if (row == kInvalidRow) flag_status(a.status, TSD_DEV_BAD_PAGE);
        S.rowaddr[slot] = row;
        S.ent_slot[m * E + e] = (uint16_t)slot;
      }
    }
  }
  const int ntiles = (nunique + kRowsPerTile - 1) / kRowsPerTile;
  // ---- 4. tile boundaries of every list: bnd[m][i] = first entry with slot >= i*R ----
  for (int i = threadIdx.x; i < nlists * (kMaxTiles + 1); i += kDecodeThreads) {
    const int m = i / (kMaxTiles + 1), tt = i % (kMaxTiles + 1);
    if (tt <= ntiles) S.bnd[m][tt] = (uint16_t)S.list_n[m];
  }
  __syncthreads();
  for (int m = 0; m < nlists; ++m) {
    const int n = S.list_n[m];
    for (int e = threadIdx.x; e < n; e += kDecodeThreads) {
      const int ti = S.ent_slot[m * E + e] / kRowsPerTile;
      const int lo = (e == 0) ? 0 : S.ent_slot[m * E + e - 1] / kRowsPerTile + 1;
      for (int tt = lo; tt <= ti; ++tt) S.bnd[m][tt] = (uint16_t)e;
    }
  }
  // prefetch the first tiles while the boundaries settle
  // (rowaddr is complete: it was written before the previous barrier)
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ntiles) load_tile(S, a.kv, s, nunique);
    cp_async_commit();
  }

  // ---- 5. lane-group roles: list m = group / P, part p = group % P ----
  const int group = threadIdx.x >> 3, l8 = threadIdx.x & 7;
  const int P = 32 / nlists;                    // parts per list (>= 1)
  const int my_list = group / P, my_part = group % P;
  const bool has_list = my_list < nlists;
  float q[16];
  SoftState st;
  soft_init(st);
  {
    const ListRef r = list_ref(a, si, g, lg, has_list ? my_list : 0);
    const float scale = a.qv.sm_scale * kLog2e;
    load_q16(a.qv, r.t, r.h, l8, scale, q);
  }

  // ---- 6. main loop over tiles ----
  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (tile + kStages - 1 < ntiles) load_tile(S, a.kv, tile + kStages - 1, nunique);
    cp_async_commit();

    const unsigned char* kbase = S.ring + (tile % kStages) * kTileBytes;
    const unsigned char* vbase = kbase + kRowsPerTile * 256;
    int ea = 0, eb = 0, first = 0, cnt = 0;
    if (has_list) {
      ea = S.bnd[my_list][tile];
      eb = S.bnd[my_list][tile + 1];
      const int n = S.list_n[my_list];
      ea = min(ea, n);
      eb = min(max(eb, ea), n);
      first = ea + ((my_part - ea) % P + P) % P;
      cnt = eb > first ? (eb - first + P - 1) / P : 0;
    }
    int nmax = cnt;
    nmax = max(nmax, __shfl_xor_sync(0xFFFFFFFFu, nmax, 8));
    nmax = max(nmax, __shfl_xor_sync(0xFFFFFFFFu, nmax, 16));
    for (int it = 0; it < nmax; ++it) {
      const int e = first + it * P;
      bool active = it < cnt;
      int r = 0;
      if (active) {
        const int slot = S.ent_slot[my_list * E + e];
        r = slot - tile * kRowsPerTile;
        if (r < 0 || r >= kRowsPerTile || S.rowaddr[slot] == kInvalidRow) {
          active = false;
          r = 0;
        }
      }
      const float s = group_dot(kbase + r * 256, l8, q);
      if (active) soft_update(st, s, vbase + r * 256, l8);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- 7. combine parts, write partial / output, merge splits ----
  float* comb = reinterpret_cast<float*>(S.ring);
  if (has_list) soft_store(comb, my_list * P + my_part, st, l8);
  __syncthreads();
  finish_lists(a, si, b, g, lg, split, nlists, P, comb, S.mx, S.lsum);
}

// ---------------------------------------------------------------------------
// Dense decode: every token of [split*W, split*W + W) for all lists of the CTA.
// Lane-groups hold 2 lists each ("sets"); the groups of a set split the tile's rows.
// ---------------------------------------------------------------------------
constexpr int kDenseHeadsPerGroup = 2;

struct DenseSmem {
  unsigned char ring[kRingBytes + 2048];   // ring; combine buffer (needs 32*2*132 floats)
  uint32_t rowaddr[kStages][kRowsPerTile];
  float mx[kMaxListsPerCta], lsum[kMaxListsPerCta];
};
static_assert(kRingBytes + 2048 >= 32 * kDenseHeadsPerGroup * kCombFloats * 4, "dense combine buffer");

__device__ __forceinline__ void dense_load_tile(DenseSmem& S, const KvView& kv, int b, int g, int tok0,
                                                int tile, int ntok, uint32_t* status) {
  const int stage = tile % kStages;
  unsigned char* base = S.ring + stage * kTileBytes;
  const int first = tok0 + tile * kRowsPerTile;
#pragma unroll
  for (int q = 0; q < (kRowsPerTile * 32) / kDecodeThreads; ++q) {
    const int id = threadIdx.x + q * kDecodeThreads;
    const int r = id >> 5, which = (id >> 4) & 1, ch = id & 15;
    const int tok = first + r;
    if (tok - tok0 < ntok) {
      const uint32_t row = kv_row(kv, b, g, tok);
      if (row != kInvalidRow) {
        const uint16_t* src = (which ? kv.v : kv.k) + (int64_t)row * kHeadDim + ch * 8;
        cp_async16(base + which * (kRowsPerTile * 256) + r * 256 + ch * 16, src);
      }
      if (which == 0 && ch == 0) {
        S.rowaddr[stage][r] = row;
        if (row == kInvalidRow) flag_status(status, TSD_DEV_BAD_PAGE);
      }
    }
  }
}

__global__ void __launch_bounds__(kDecodeThreads, 2) dense_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DenseSmem& S = *reinterpret_cast<DenseSmem*>(smem_raw);

  const int split = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, split == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;

  const int tok0 = split * a.span;
  int ntok = si.len - tok0;
  if (ntok > a.span) ntok = a.span;
  if (ntok < 0) ntok = 0;
  const int ntiles = (ntok + kRowsPerTile - 1) / kRowsPerTile;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ntiles) dense_load_tile(S, a.kv, b, g, tok0, s, ntok, a.status);
    cp_async_commit();
  }

  const int group = threadIdx.x >> 3, l8 = threadIdx.x & 7;
  const int nsets = (nlists + kDenseHeadsPerGroup - 1) / kDenseHeadsPerGroup;
  const int PG = 32 / nsets;   // groups per set (nsets <= 16 -> PG >= 2)
  const int my_set = group / PG, my_part = group % PG;
  const bool has_set = my_set < nsets;

  float q[kDenseHeadsPerGroup][16];
  SoftState st[kDenseHeadsPerGroup];
  int kvlen[kDenseHeadsPerGroup];
  const float scale = a.qv.sm_scale * kLog2e;
#pragma unroll
  for (int hh = 0; hh < kDenseHeadsPerGroup; ++hh) {
    soft_init(st[hh]);
    const int m = my_set * kDenseHeadsPerGroup + hh;
    const ListRef r = list_ref(a, si, g, lg, (has_set && m < nlists) ? m : 0);
    kvlen[hh] = (has_set && m < nlists) ? r.kvlen : 0;
    load_q16(a.qv, r.t, r.h, l8, scale, q[hh]);
  }

  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (tile + kStages - 1 < ntiles) dense_load_tile(S, a.kv, b, g, tok0, tile + kStages - 1, ntok, a.status);
    cp_async_commit();

    const int stage = tile % kStages;
    const unsigned char* kbase = S.ring + stage * kTileBytes;
    const unsigned char* vbase = kbase + kRowsPerTile * 256;
    const int rows = min(kRowsPerTile, ntok - tile * kRowsPerTile);
    // rows r = my_part, my_part + PG, ...: the loop bound is the same for every group
    for (int r0 = 0; r0 < kRowsPerTile; r0 += PG) {
      const int r = r0 + my_part;
      const bool row_ok = has_set && r < rows && S.rowaddr[stage][r < kRowsPerTile ? r : 0] != kInvalidRow;
      const int rr = (r < kRowsPerTile) ? r : 0;
      const int tok = tok0 + tile * kRowsPerTile + rr;
      const unsigned char* krow = kbase + rr * 256;
      uint4 k0 = *reinterpret_cast<const uint4*>(krow + 16 * l8);
      uint4 k1 = *reinterpret_cast<const uint4*>(krow + 128 + 16 * l8);
      float kf[16];
      unpack8(k0, kf);
      unpack8(k1, kf + 8);
      float s[kDenseHeadsPerGroup];
#pragma unroll
      for (int hh = 0; hh < kDenseHeadsPerGroup; ++hh) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          s0 = fmaf(q[hh][j], kf[j], s0);
          s1 = fmaf(q[hh][8 + j], kf[8 + j], s1);
        }
        s[hh] = s0 + s1;
      }
#pragma unroll
      for (int hh = 0; hh < kDenseHeadsPerGroup; ++hh) {
        s[hh] += __shfl_xor_sync(0xFFFFFFFFu, s[hh], 1);
        s[hh] += __shfl_xor_sync(0xFFFFFFFFu, s[hh], 2);
        s[hh] += __shfl_xor_sync(0xFFFFFFFFu, s[hh], 4);
      }
      if (row_ok) {
#pragma unroll
        for (int hh = 0; hh < kDenseHeadsPerGroup; ++hh)
          if (tok < kvlen[hh]) soft_update(st[hh], s[hh], vbase + rr * 256, l8);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  float* comb = reinterpret_cast<float*>(S.ring);
  if (has_set) {
#pragma unroll
    for (int hh = 0; hh < kDenseHeadsPerGroup; ++hh) {
      const int m = my_set * kDenseHeadsPerGroup + hh;
      if (m < nlists) soft_store(comb, m * PG + my_part, st[hh], l8);
    }
  }
  __syncthreads();
  finish_lists(a, si, b, g, lg, split, nlists, PG, comb, S.mx, S.lsum);
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_sparse_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream) {
  const size_t smem = sizeof(SparseSmem);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(a.nsplit, hkv * a.list_groups, batch);
  sparse_decode_kernel<<<grid, kDecodeThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dense_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream) {
  const size_t smem = sizeof(DenseSmem);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(dense_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(a.nsplit, hkv * a.list_groups, batch);
  dense_decode_kernel<<<grid, kDecodeThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tsd
