// Sparse and dense decode attention kernels for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?",
// gist.science summary, section 2 "Hardware implementation" and section 3.C):
// for each (query token t, q head h) attend only to the K/V rows named by its
// index list -- which may differ per token, per query and per head -- so that
// the bytes read fall from O(N d) to O(k d).  Dense decode attends to every row.
//
// Sparse decode: one warp per task (a chunk of one list); 16-row K/V tiles gathered through a
// per-warp cp.async ring; q K^T and P V of each tile on the tensor cores; per-list split-K
// merge in the CTA, then by the last CTA of the list to finish.
// Dense decode: one CTA per (sequence, kv head, list group, window of W tokens); 64-token
// K/V tiles arrive by TMA in a 2-stage shared-memory ring and q K^T and P V run on the
// tensor cores; CTA-level partials are merged by the last CTA of the unit.
// No kernel ever waits on another CTA: merges are done by whichever arrives last.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "tsd_args.h"
#include "tsd_common.cuh"
#include "tsd_kvtile.cuh"

namespace tsd {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kCombFloats = 132;                             // m, l, pad, pad, acc[128]


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
      // 8 splits at a time with independent loads (one L2 round trip per 8 splits)
      for (int c0 = 0; c0 < a.nsplit; c0 += 8) {
        float mm[8], aa[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u;
          mm[u] = c < a.nsplit ? __ldcg(&a.part_ml[pbase + c]).x : -CUDART_INF_F;
          aa[u] = c < a.nsplit ? __ldcg(&a.part_acc[(pbase + c) * kHeadDim + d]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = fast_exp2(mm[u] - mx);   // 0 for empty splits (mm = -inf)
          A = fmaf(w, aa[u], A);
        }
      }
    }
    store_out(a, r.t, r.h, d, L > 0.f ? A / L : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Sparse decode
// ---------------------------------------------------------------------------
// Design, from measurements on B200:
//  * One warp per task: a chunk of E entries of one list (token x q head).  The plan sizes E
//    so that the grid fits one wave of resident CTAs; the CTA's warps take consecutive
//    chunks of a list, which are combined in shared memory before anything leaves the CTA.
//  * The task's rows are gathered 16 at a time (a tile: 16 K rows then 16 V rows, 256 bytes
//    each) into a per-warp ring of kSpStages tiles in shared memory with 16-byte cp.async
//    copies; rows that are not there (padding, -1 entries, bad pages) are zero-filled by the
//    same copies.  Entries are resolved a window of 32 (one per lane) at a time, and two
//    windows ahead: the page-table rows of window w + 2 and the raw indices of window w + 3
//    are in flight while window w's tiles are consumed, so a tile's rows are known a whole
//    window before its copies are issued.
//  * Both contractions of a tile run on the tensor cores (mma.m16n8k16, bf16 in, fp32
//    accumulate), with the unused columns of the n = 8 operand carrying a second bf16 part:
//      scores  S(16 rows x 8) = K(16 x 128) . [q_hi, q_lo, 0 ...]    (columns 0 and 1 summed)
//      output  O^T(128 x 8) += V^T(128 x 16) . [P_hi, P_lo, 0 ...]   (columns 0 and 1 summed)
//    where x_hi = bf16(x) and x_lo = bf16(x - x_hi), so an fp32 q and the fp32 softmax
//    weights enter with about 16 significant bits.  Against one CUDA-core dot product per
//    row and half-warp this cut the executed instructions per gathered row from 49 to 28.
//  * Online softmax in base-2 units with a lazily moved reference: the running maximum is
//    only raised (and the state rescaled) when a tile exceeds it by more than 2^8, so most
//    tiles skip the rescale; weights then stay below 2^8.
// The CTA's per-task states of a list are combined in shared memory; each CTA then writes one
// partial per list, and the last CTA of a list to arrive (a per-list counter) merges them with
// log-sum-exp.  A list held by one CTA alone is written directly.
constexpr int kSpWarps = kSpTasksPerCta;
constexpr int kSpThreads = 32 * kSpWarps;
constexpr int kSpTileRows = 16;
constexpr int kSpHalfBytes = kSpTileRows * kHeadDim * 2;   // 16 rows of K (or V): 4 KB
constexpr int kSpTileBytes = 2 * kSpHalfBytes;
constexpr size_t kSpRingBytes = (size_t)kSpWarps * kSpStages * kSpTileBytes;
constexpr int kSpPtEntries = 2048;                     // page-table row cached in shared memory up to this length
constexpr size_t kSpSmemBytes = kSpRingBytes + kSpPtEntries * sizeof(int32_t);
constexpr float kSpLazyMax = 8.f;   // base-2 units the running maximum may lag behind
static_assert(kSpStages >= 2 && kSpStages <= 3, "the ring looks at most one window (two tiles) ahead");
static_assert(kSpCtasPerSm * (kSpSmemBytes + 4096) <= 228 * 1024, "resident sparse CTAs per SM");

// Byte offset of 16-byte chunk c of row r in a tile of 256-byte rows, the chunk index XOR-ed
// with (r mod 8): the 8 rows one ldmatrix phase reads fall in 8 different bank groups.
__device__ __forceinline__ uint32_t sp_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4)); }

// 16-byte cp.async that writes zeros (and reads nothing) when !valid.
__device__ __forceinline__ void cp_async16_zfill(uint32_t smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem), "l"(gmem), "r"(valid ? 16 : 0)
               : "memory");
}

// Four consecutive output dims [d, d + 4) of (token t, q head h).
__device__ __forceinline__ void store_out4(const DecodeArgs& a, int t, int h, int d, float4 v) {
  const int64_t o = ((int64_t)t * a.qv.hq + h) * kHeadDim + d;
  if (a.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + o) = v;
  } else {
    uint2 w;
    w.x = (uint32_t)f32_to_bf16_rne(v.x) | ((uint32_t)f32_to_bf16_rne(v.y) << 16);
    w.y = (uint32_t)f32_to_bf16_rne(v.z) | ((uint32_t)f32_to_bf16_rne(v.w) << 16);
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) + o) = w;
  }
}

// End of a list's work in one CTA, by one warp (lane l holding output dims [4l, 4l + 4)): a
// list whose chunks all ran in this CTA is written directly; otherwise this CTA's partial
// state (partial c of C) is stored, and the last CTA of the list to arrive (per-list counter)
// merges the C partials with log-sum-exp.
__device__ __forceinline__ void finish_list(const DecodeArgs& a, int64_t list_id, int t, int h, int C, int c,
                                            float m_run, float l_run, float4 acc, int l) {
  if (C == 1) {
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    store_out4(a, t, h, 4 * l, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    if (l == 0 && a.lse != nullptr) a.lse[list_id] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -CUDART_INF_F;
    return;
  }
  const int64_t pidx = list_id * a.nsplit + c;
  if (l == 0) a.part_ml[pidx] = make_float2(m_run, l_run);
  reinterpret_cast<float4*>(a.part_acc + pidx * kHeadDim)[l] = acc;
  __threadfence();
  __syncwarp();
  uint32_t prev = 0;
  if (l == 0) {
    prev = atomicAdd(a.counters + list_id, 1u);
    if (prev == (uint32_t)(C - 1)) atomicExch(a.counters + list_id, 0u);   // leave it zero for the next call
  }
  prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
  if (prev != (uint32_t)(C - 1)) return;
  __threadfence();
  // last CTA of the list: max and sum over the C partials (lanes over partials), then 4 dims
  // per lane with 8 independent loads in flight
  const float2* ml = a.part_ml + list_id * a.nsplit;
  float mx = -CUDART_INF_F;
  for (int i = l; i < C; i += 32) mx = fmaxf(mx, __ldcg(&ml[i]).x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  float L = 0.f;
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -CUDART_INF_F) {
    for (int i = l; i < C; i += 32) {
      const float2 x = __ldcg(&ml[i]);
      L = fmaf(fast_exp2(x.x - mx), x.y, L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
    const float4* src = reinterpret_cast<const float4*>(a.part_acc + list_id * a.nsplit * kHeadDim) + l;
    for (int c0 = 0; c0 < C; c0 += 8) {
      float w[8];
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int cc = c0 + u < C ? c0 + u : C - 1;
        w[u] = c0 + u < C ? fast_exp2(__ldcg(&ml[cc]).x - mx) : 0.f;
        x[u] = __ldcg(src + (int64_t)cc * (kHeadDim / 4));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        r.x = fmaf(w[u], x[u].x, r.x); r.y = fmaf(w[u], x[u].y, r.y);
        r.z = fmaf(w[u], x[u].z, r.z); r.w = fmaf(w[u], x[u].w, r.w);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  store_out4(a, t, h, 4 * l, make_float4(r.x * inv, r.y * inv, r.z * inv, r.w * inv));
  if (l == 0 && a.lse != nullptr) a.lse[list_id] = L > 0.f ? (mx + log2f(L)) * kLn2 : -CUDART_INF_F;
}

template <bool WEIGHTED>
__global__ void __launch_bounds__(kSpThreads, kSpCtasPerSm) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char sp_ring[];   // [warp][kSpStages][K rows, V rows]
  pdl_wait();   // a dependent launch (after the selection that wrote idx) starts here
  // task states of the CTA's warps, combined per list before anything leaves the CTA
  __shared__ float2 s_ml[kSpWarps];
  __shared__ __align__(16) float s_acc[kSpWarps][kHeadDim];
  __shared__ int64_t s_list[kSpWarps];
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int G = a.qv.hq / a.kv.hkv;
  const int M = a.lists_per_cta;   // list slots per (sequence, kv head): G x max tokens per sequence
  const int C = a.nsplit;          // tasks (chunks) per list
  const int E = a.span;            // entries per task
  // tasks are numbered (sequence, kv head, list, chunk): a CTA's warps hold consecutive
  // chunks of a list
  const int64_t task = (int64_t)blockIdx.x * kSpWarps + warp;
  const int64_t total = (int64_t)a.kv.batch * a.kv.hkv * M * C;
  const int64_t tk = task < total ? task : total - 1;
  const int c = (int)(tk % C);
  int64_t rest = tk / C;
  const int m = (int)(rest % M);
  rest /= M;
  const int g = (int)(rest % a.kv.hkv);
  const int b = (int)(rest / a.kv.hkv);

  // The gather's first rows wait on a chain of dependent reads (sequence -> index -> page ->
  // row).  Without q_indptr a sequence has the single query token t = b, so the list is known
  // before the sequence descriptor arrives: the first four windows of raw indices are loaded
  // alongside it.
  const int e0 = c * E;
  const int e1 = min(e0 + E, a.k_max);
  const int nwin = (e1 - e0 + 31) >> 5;   // windows of 32 entries (two tiles), one per lane
  const bool early = a.qv.q_indptr == nullptr && task < total && m < G && b < a.qv.num_tokens;
  int32_t raw0[4];
  int32_t prev0 = -1;
  if (early) {
    const int32_t* lst = a.idx + ((int64_t)b * a.qv.hq + g * G + m) * a.k_max;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int e = e0 + 32 * w + lane;
      raw0[w] = (w < nwin && e < e1) ? __ldg(lst + e) : -1;
    }
    if (lane == 0 && e0 > 0) prev0 = __ldg(lst + e0 - 1);
  }
  // the sequence descriptor's reads are in flight together with the index loads above and the
  // page-table copy below; it is checked after both
  const SeqRaw sraw = seq_load(a.kv, a.qv, b);
  // When the CTA's tasks all belong to one sequence and its page-table row is short, the row
  // is copied into shared memory alongside the index loads: the page lookups of the gather then
  // cost no global round trip.
  const int64_t per_seq = (int64_t)a.kv.hkv * M * C;
  const int64_t t_first = (int64_t)blockIdx.x * kSpWarps;
  const int64_t t_last = (t_first + kSpWarps < total ? t_first + kSpWarps : total) - 1;
  const bool pt_smem = a.kv.page_table != nullptr && a.kv.max_pages <= kSpPtEntries && t_first / per_seq == t_last / per_seq;
  int32_t* s_pt = reinterpret_cast<int32_t*>(sp_ring + kSpRingBytes);
  if (pt_smem) {
    const int32_t* src = a.kv.page_table + (t_first / per_seq) * a.kv.max_pages;
    for (int i = threadIdx.x; i < a.kv.max_pages; i += kSpThreads) s_pt[i] = __ldg(src + i);
    __syncthreads();
  }
  const SeqInfo si = seq_check(a.kv, a.qv, sraw, a.status, task == tk && c == 0 && g == 0 && m == 0 && lane == 0);
  const int j = m / G;
  const bool valid = task < total && j < si.n;   // no list for slots past this sequence's tokens
  const int t = si.t0 + j, h = g * G + (m - j * G);
  const int64_t list_id = valid ? (int64_t)t * a.qv.hq + h : -1;
  float m_run = -CUDART_INF_F, l_run = 0.f;   // l_run: this lane's share of the sum
  float o[8][4];                              // O^T accumulators, m-tile i = dims [16i, 16i + 16)
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  if (valid) {
    const int kvlen = kv_len_of(a.qv, si, j);
    const float scale = a.qv.sm_scale * kLog2e;   // dots -> base-2 softmax units
    // q as the B operand of the score MMA (k = dims, n = columns): lane 4n + i holds column n,
    // dims 16ks + 2i, +1 and 16ks + 2i + 8, +9; column 0 = bf16(q), column 1 = q - bf16(q)
    uint32_t qb[8][2];
    {
      const int col = lane >> 2, i2 = 2 * (lane & 3);
      const int64_t qb0 = list_id * kHeadDim;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qb[ks][0] = qb[ks][1] = 0u;
        if (col < 2) {
          const int d0 = 16 * ks + i2;
          float x0, x1, y0, y1;
          if (a.qv.q_f32) {
            const float* qp = reinterpret_cast<const float*>(a.qv.q) + qb0;
            const float2 u = __ldg(reinterpret_cast<const float2*>(qp + d0));
            const float2 v = __ldg(reinterpret_cast<const float2*>(qp + d0 + 8));
            x0 = u.x; x1 = u.y; y0 = v.x; y1 = v.y;
          } else {
            const uint16_t* qp = reinterpret_cast<const uint16_t*>(a.qv.q) + qb0;
            const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(qp + d0));
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(qp + d0 + 8));
            x0 = bf16lo(u); x1 = bf16hi(u); y0 = bf16lo(v); y1 = bf16hi(v);
          }
          uint32_t h0, l0, h1, l1;
          split_bf16(x0, x1, h0, l0);
          split_bf16(y0, y1, h1, l1);
          qb[ks][0] = col == 0 ? h0 : l0;
          qb[ks][1] = col == 0 ? h1 : l1;
        }
      }
    }

    const int32_t* lst = a.idx + list_id * a.k_max;
    const int ntile = (e1 - e0 + kSpTileRows - 1) / kSpTileRows;
    uint32_t bad = 0;
    auto load_raw = [&](int wi) -> int32_t {   // raw index of entry e0 + 32 wi + lane, -1 past the end
      const int e = e0 + 32 * wi + lane;
      return (wi < nwin && e < e1) ? __ldg(lst + e) : -1;
    };
    auto load_lw = [&](int wi) -> float {      // its weight, base-2 units
      const int e = e0 + 32 * wi + lane;
      return (WEIGHTED && wi < nwin && e < e1) ? __ldg(a.logw + list_id * a.k_max + e) * kLog2e : 0.f;
    };
    // window wi's raw indices -> physical rows, with the order / range / page checks; `prev`
    // is (in lane 0) the raw index of the entry before the window
    auto resolve = [&](int wi, int32_t v, int32_t prev) -> uint32_t {
      const int e = e0 + 32 * wi + lane;
      uint32_t before = __shfl_up_sync(FULL, (uint32_t)v, 1);
      if (lane == 0) before = (uint32_t)prev;
      const bool in = wi < nwin && e < e1;
      if (in && e > 0 && (uint32_t)v < before) bad |= TSD_DEV_UNSORTED;
      if (in && (v < -1 || v >= kvlen)) bad |= TSD_DEV_BAD_INDEX;
      uint32_t row = kInvalidRow;
      if (in && v >= 0 && v < kvlen) {
        if (pt_smem) {   // the same mapping as kv_row, from the shared-memory copy
          const int32_t page = s_pt[v >> a.kv.page_shift];
          if (page >= 0 && (int64_t)page < a.kv.num_pages)
            row = (uint32_t)((((int64_t)page * a.kv.hkv + g) << a.kv.page_shift) | (v & ((1 << a.kv.page_shift) - 1)));
        } else {
          row = kv_row(a.kv, b, g, v);
        }
        if (row == kInvalidRow) bad |= TSD_DEV_BAD_PAGE;
      }
      return row;
    };
    // tile p (0 or 1) of the window whose rows are `rows` -> ring stage `stage`: lane l copies
    // chunk l mod 16 of rows 2i + l / 16
    const uint32_t ring = smem_u32(sp_ring) + (uint32_t)(warp * kSpStages * kSpTileBytes);
    auto issue = [&](uint32_t rows, int p, int stage) {
      const uint32_t st = ring + (uint32_t)(stage * kSpTileBytes);
      const int cc = lane & 15;
#pragma unroll
      for (int i = 0; i < kSpTileRows / 2; ++i) {
        const int r = 2 * i + (lane >> 4);
        const uint32_t rr = __shfl_sync(FULL, rows, 16 * p + r);
        const bool ok = rr != kInvalidRow;
        const int64_t off = ok ? (int64_t)rr * kHeadDim : 0;
        const uint32_t so = sp_off(r, cc);
        cp_async16_zfill(st + so, reinterpret_cast<const uint4*>(a.kv.k + off) + cc, ok);
        cp_async16_zfill(st + kSpHalfBytes + so, reinterpret_cast<const uint4*>(a.kv.v + off) + cc, ok);
      }
      cp_async_commit();
    };

    // rows of windows wi, wi + 1 and wi + 2 resolved, raw indices of window wi + 3 loaded: a
    // window's page-table reads are issued a whole window before its first tile is issued
    if (!early) {
#pragma unroll
      for (int w = 0; w < 4; ++w) raw0[w] = load_raw(w);
      if (lane == 0 && e0 > 0) prev0 = __ldg(lst + e0 - 1);
    }
    const int32_t v0 = raw0[0], v1 = raw0[1], v2 = raw0[2];
    int32_t v3 = raw0[3];
    float lw_cur = load_lw(0), lw_nxt = load_lw(1), lw_n2 = load_lw(2), lw_n3 = load_lw(3);
    uint32_t row_cur = resolve(0, v0, prev0);
    int32_t last = __shfl_sync(FULL, v0, 31);
    uint32_t row_nxt = resolve(1, v1, last);
    last = __shfl_sync(FULL, v1, 31);
    uint32_t row_n2 = resolve(2, v2, last);
    last = __shfl_sync(FULL, v2, 31);
#pragma unroll
    for (int ta = 0; ta < kSpStages - 1; ++ta) {   // tiles 0 .. kSpStages - 2, all in window 0
      if (ta < ntile) issue(row_cur, ta, ta); else cp_async_commit();
    }
    // lanes 4i hold the scores of tile rows i and i + 8
    const int gi = lane >> 2;
    const bool scol = (lane & 3) == 0;
    // P^T as the B operand of the output MMA: lane 4n + i needs rows 2i, 2i + 1 (from lanes
    // 8i, 8i + 4, first score) and 2i + 8, 2i + 9 (second score); n = 0 takes bf16(P), n = 1 the rest
    const int psrc = 8 * (lane & 3);
    // ldmatrix lane addresses: K (non-transposed) rows l mod 16, chunk half l / 16; V
    // (transposed) rows (l mod 8) + 8 (l / 16), chunk half (l / 8) mod 2
    const int kr = lane & 15, kh = lane >> 4;
    const int vr = (lane & 7) + 8 * (lane >> 4), vh = (lane >> 3) & 1;
    int stage = 0;
    for (int wi = 0; wi < nwin; ++wi) {
      const uint32_t vmask = __ballot_sync(FULL, row_cur != kInvalidRow);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int tt = 2 * wi + p;
        if (tt >= ntile) break;
        // keep kSpStages - 1 tiles ahead of the one consumed
        {
          const int ta = tt + kSpStages - 1;
          const int ap = (p + kSpStages - 1) & 1;
          const bool next_win = ((p + kSpStages - 1) >> 1) != 0;
          const int ast = stage == 0 ? kSpStages - 1 : stage - 1;
          __syncwarp();
          if (ta < ntile) issue(next_win ? row_nxt : row_cur, ap, ast); else cp_async_commit();
        }
        cp_async_wait<kSpStages - 1>();
        __syncwarp();   // every lane's copies of this tile have landed
        const uint32_t st = ring + (uint32_t)(stage * kSpTileBytes);
        const uint32_t tmask = (vmask >> (16 * p)) & 0xFFFFu;
        // scores: two accumulator chains over the 8 k-steps
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t af[4];
          ldsm_x4(st + sp_off(kr, 2 * ks + kh), af[0], af[1], af[2], af[3]);
          mma_bf16((ks & 1) ? d1 : d0, af, qb[ks][0], qb[ks][1]);
        }
        float s0 = ((d0[0] + d1[0]) + (d0[1] + d1[1])) * scale;
        float s1 = ((d0[2] + d1[2]) + (d0[3] + d1[3])) * scale;
        if (WEIGHTED) {   // entry weights: p_i = w_i exp(s_i), with ln w_i in base-2 units
          s0 += __shfl_sync(FULL, lw_cur, 16 * p + gi);
          s1 += __shfl_sync(FULL, lw_cur, 16 * p + gi + 8);
        }
        s0 = (scol && ((tmask >> gi) & 1u)) ? s0 : -CUDART_INF_F;
        s1 = (scol && ((tmask >> (gi + 8)) & 1u)) ? s1 : -CUDART_INF_F;
        float mt = fmaxf(s0, s1);
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
        mt = __shfl_sync(FULL, mt, 0);
        if (mt != -CUDART_INF_F) {   // uniform over the warp
          if (mt > m_run + kSpLazyMax) {   // move the reference (always on the first valid tile)
            const float alpha = fast_exp2(m_run - mt);
            l_run *= alpha;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              o[i][0] *= alpha; o[i][1] *= alpha; o[i][2] *= alpha; o[i][3] *= alpha;
            }
            m_run = mt;
          }
          const float p0 = fast_exp2(s0 - m_run), p1 = fast_exp2(s1 - m_run);   // 0 for masked rows
          l_run += p0 + p1;
          const float x0 = __shfl_sync(FULL, p0, psrc), x1 = __shfl_sync(FULL, p0, psrc + 4);
          const float y0 = __shfl_sync(FULL, p1, psrc), y1 = __shfl_sync(FULL, p1, psrc + 4);
          uint32_t h0, l0, h1, l1;
          split_bf16(x0, x1, h0, l0);
          split_bf16(y0, y1, h1, l1);
          const uint32_t pb0 = lane < 4 ? h0 : (lane < 8 ? l0 : 0u);
          const uint32_t pb1 = lane < 4 ? h1 : (lane < 8 ? l1 : 0u);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t af[4];
            ldsm_x4_t(st + kSpHalfBytes + sp_off(vr, 2 * i + vh), af[0], af[1], af[2], af[3]);
            mma_bf16(o[i], af, pb0, pb1);
          }
        }
        stage = stage + 1 == kSpStages ? 0 : stage + 1;
      }
      // rotate: window wi + 1 becomes current, resolve window wi + 3, load window wi + 4
      row_cur = row_nxt;
      row_nxt = row_n2;
      row_n2 = resolve(wi + 3, v3, last);
      last = __shfl_sync(FULL, v3, 31);
      v3 = load_raw(wi + 4);
      if (WEIGHTED) {
        lw_cur = lw_nxt;
        lw_nxt = lw_n2;
        lw_n2 = lw_n3;
        lw_n3 = load_lw(wi + 4);
      }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) bad |= __shfl_xor_sync(FULL, bad, o2);
    if (lane == 0 && bad) flag_status(a.status, bad);
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) l_run += __shfl_xor_sync(FULL, l_run, o2);
    l_run = __shfl_sync(FULL, l_run, 0);
  }

  // task states -> shared memory (lanes 4i hold dims 16k + i and 16k + i + 8, columns 0 + 1)
  if (lane == 0) {
    s_ml[warp] = make_float2(m_run, l_run);
    s_list[warp] = list_id;
  }
  if ((lane & 3) == 0) {
    const int i = lane >> 2;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      s_acc[warp][16 * k + i] = o[k][0] + o[k][1];
      s_acc[warp][16 * k + i + 8] = o[k][2] + o[k][3];
    }
  }
  __syncthreads();
  if (!valid || (warp > 0 && s_list[warp - 1] == list_id)) return;   // not the first chunk of its list here
  float mm = m_run, ll = l_run;
  float4 acc = *reinterpret_cast<const float4*>(&s_acc[warp][4 * lane]);
  for (int w2 = warp + 1; w2 < kSpWarps && s_list[w2] == list_id; ++w2) {
    const float2 x = s_ml[w2];
    const float mn = fmaxf(mm, x.x);
    if (mn == -CUDART_INF_F) continue;
    const float wa = fast_exp2(mm - mn), wb = fast_exp2(x.x - mn);
    const float4 y = *reinterpret_cast<const float4*>(&s_acc[w2][4 * lane]);
    ll = ll * wa + x.y * wb;
    acc.x = acc.x * wa + y.x * wb; acc.y = acc.y * wa + y.y * wb;
    acc.z = acc.z * wa + y.z * wb; acc.w = acc.w * wa + y.w * wb;
    mm = mn;
  }
  // partials of the list = CTAs that hold one of its chunks; this CTA's partial index
  const int64_t first = (((int64_t)b * a.kv.hkv + g) * M + m) * C;
  const int64_t fc = first / kSpWarps, lc = (first + C - 1) / kSpWarps;
  finish_list(a, list_id, t, h, (int)(lc - fc + 1), (int)((int64_t)blockIdx.x - fc), mm, ll, acc, lane);
}

// ---------------------------------------------------------------------------
// Sparse decode, persistent form
// ---------------------------------------------------------------------------
// The one-task-per-warp kernel above fits its grid to one wave of resident CTAs.  When the
// lists outnumber that wave (many decode tokens, long and unequal lists), it runs several
// waves whose CTAs each pay the dependent start (sequence -> index -> page -> row) again, and
// its last wave runs with idle SMs.  This form keeps kSsCtasPerSm CTAs on every SM for the
// whole call instead.  Every warp takes (list, chunk) tasks from a counter in the workspace
// until none is left, and its pipeline runs straight across task boundaries:
//   S3  raw indices of a window (32 entries, one per lane) -- a new task is fetched here;
//   S2  the window resolved to physical rows (order / range / page checks);
//   S1  the window whose two 16-row tiles are being copied into the ring;
//   S0  the window whose tiles are consumed (q K^T, online softmax, P V on the tensor cores).
// A task's descriptor (list, chunk, bounds) and its q row sit in a per-warp shared-memory slot
// from the fetch until the task finishes.  A chunk whose first entry is -1 lies past the end
// of its list and is skipped at the fetch; a window whose entries are all -1 ends its task.
// Split-K partials: a list of C > 1 chunks has its non-empty chunks write partials and arrive
// on the list's counter; the chunk that holds the list's last entry adds its chunk count in
// the counter's upper half, so the arrival that completes the count -- whichever it is --
// merges the partials.  The last warp of the grid to finish clears the counters.
constexpr int kSsWarps = kSsWarpsPerCta;
constexpr int kSsThreads = 32 * kSsWarps;
constexpr int kSsSlots = 4;                                   // task slots per warp
constexpr uint32_t kTagSlot = 3u;                            // slot bits of a window tag
constexpr uint32_t kTagFirst = 1u << 8;                      // first window of its task
constexpr uint32_t kTagLast = 1u << 9;                       // last window of its task
constexpr uint32_t kTagBubble = 1u << 10;                    // a window with no entries
constexpr uint32_t kTagEnd = 1u << 11;                       // the warp has no task left
static_assert(kSsSlots - 1 == (int)kTagSlot, "slot bits");

struct SsDesc {
  int list, c, e1, kvlen, b, g, pad0, pad1;
};
constexpr size_t kSsRingBytes = (size_t)kSsWarps * kSpStages * kSpTileBytes;
constexpr size_t kSsQBytes = (size_t)kSsWarps * kSsSlots * 512;   // fp32 q rows at most
constexpr size_t kSsDescBytes = (size_t)kSsWarps * kSsSlots * sizeof(SsDesc);
constexpr size_t kSsAccBytes = (size_t)kSsWarps * kHeadDim * sizeof(float);
constexpr size_t kSsSmemBytes = kSsRingBytes + kSsQBytes + kSsDescBytes + kSsAccBytes;
static_assert(kSsCtasPerSm * (kSsSmemBytes + 2048) <= 228 * 1024, "resident persistent CTAs per SM");

// One 16-row tile of a list (ring stage `st`: K rows then V rows, chunk-swizzled): scores on
// the tensor cores, the lazily moved online softmax, and O^T += V^T P^T.  `tmask` holds the
// tile's valid rows; lw (weighted form) is this lane's entry weight of the tile's window.
template <bool WEIGHTED>
__device__ __forceinline__ void sp_tile(uint32_t st, uint32_t tmask, const uint32_t (&qb)[8][2], float scale,
                                        float lw, int p, float& m_run, float& l_run, float (&o)[8][4]) {
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int gi = lane >> 2;
  const bool scol = (lane & 3) == 0;
  const int psrc = 8 * (lane & 3);
  const int kr = lane & 15, kh = lane >> 4;
  const int vr = (lane & 7) + 8 * (lane >> 4), vh = (lane >> 3) & 1;
  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t af[4];
    ldsm_x4(st + sp_off(kr, 2 * ks + kh), af[0], af[1], af[2], af[3]);
    mma_bf16((ks & 1) ? d1 : d0, af, qb[ks][0], qb[ks][1]);
  }
  float s0 = ((d0[0] + d1[0]) + (d0[1] + d1[1])) * scale;
  float s1 = ((d0[2] + d1[2]) + (d0[3] + d1[3])) * scale;
  if (WEIGHTED) {
    s0 += __shfl_sync(FULL, lw, 16 * p + gi);
    s1 += __shfl_sync(FULL, lw, 16 * p + gi + 8);
  }
  s0 = (scol && ((tmask >> gi) & 1u)) ? s0 : -CUDART_INF_F;
  s1 = (scol && ((tmask >> (gi + 8)) & 1u)) ? s1 : -CUDART_INF_F;
  float mt = fmaxf(s0, s1);
  mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
  mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
  mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
  mt = __shfl_sync(FULL, mt, 0);
  if (mt == -CUDART_INF_F) return;   // uniform over the warp
  if (mt > m_run + kSpLazyMax) {
    const float alpha = fast_exp2(m_run - mt);
    l_run *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[i][0] *= alpha; o[i][1] *= alpha; o[i][2] *= alpha; o[i][3] *= alpha;
    }
    m_run = mt;
  }
  const float p0 = fast_exp2(s0 - m_run), p1 = fast_exp2(s1 - m_run);
  l_run += p0 + p1;
  const float x0 = __shfl_sync(FULL, p0, psrc), x1 = __shfl_sync(FULL, p0, psrc + 4);
  const float y0 = __shfl_sync(FULL, p1, psrc), y1 = __shfl_sync(FULL, p1, psrc + 4);
  uint32_t h0, l0, h1, l1;
  split_bf16(x0, x1, h0, l0);
  split_bf16(y0, y1, h1, l1);
  const uint32_t pb0 = lane < 4 ? h0 : (lane < 8 ? l0 : 0u);
  const uint32_t pb1 = lane < 4 ? h1 : (lane < 8 ? l1 : 0u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t af[4];
    ldsm_x4_t(st + kSpHalfBytes + sp_off(vr, 2 * i + vh), af[0], af[1], af[2], af[3]);
    mma_bf16(o[i], af, pb0, pb1);
  }
}

// Merge the `ce` split partials of list `list_id` (lane l: output dims [4l, 4l + 4)) and write
// out and lse.
__device__ __forceinline__ void merge_partials_of_list(const DecodeArgs& a, int64_t list_id, int ce, int l) {
  const float2* ml = a.part_ml + list_id * a.nsplit;
  float mx = -CUDART_INF_F;
  for (int i = l; i < ce; i += 32) mx = fmaxf(mx, __ldcg(&ml[i]).x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  float L = 0.f;
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -CUDART_INF_F) {
    for (int i = l; i < ce; i += 32) {
      const float2 x = __ldcg(&ml[i]);
      L = fmaf(fast_exp2(x.x - mx), x.y, L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
    const float4* src = reinterpret_cast<const float4*>(a.part_acc + list_id * a.nsplit * kHeadDim) + l;
    for (int c0 = 0; c0 < ce; c0 += 8) {
      float w[8];
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int cc = c0 + u < ce ? c0 + u : ce - 1;
        const float m = __ldcg(&ml[cc]).x;
        w[u] = (c0 + u < ce && m != -CUDART_INF_F) ? fast_exp2(m - mx) : 0.f;
        x[u] = __ldcg(src + (int64_t)cc * (kHeadDim / 4));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (w[u] == 0.f) continue;   // an empty partial's row is never read into the sum
        r.x = fmaf(w[u], x[u].x, r.x); r.y = fmaf(w[u], x[u].y, r.y);
        r.z = fmaf(w[u], x[u].z, r.z); r.w = fmaf(w[u], x[u].w, r.w);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int t = (int)(list_id / a.qv.hq), h = (int)(list_id % a.qv.hq);
  store_out4(a, t, h, 4 * l, make_float4(r.x * inv, r.y * inv, r.z * inv, r.w * inv));
  if (l == 0 && a.lse != nullptr) a.lse[list_id] = L > 0.f ? (mx + log2f(L)) * kLn2 : -CUDART_INF_F;
}

template <bool WEIGHTED>
__global__ void __launch_bounds__(kSsThreads, kSsCtasPerSm) sparse_stream_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char ss_smem[];
  pdl_wait();   // a dependent launch (after the selection that wrote idx) starts here
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int G = a.qv.hq / a.kv.hkv;
  const int M = a.lists_per_cta;   // list slots per (sequence, kv head)
  const int C = a.nsplit;          // chunks per list
  const int E = a.span;            // entries per chunk, a multiple of 32
  const int64_t total = (int64_t)a.kv.batch * a.kv.hkv * M * C;
  const uint32_t ring = smem_u32(ss_smem) + (uint32_t)(warp * kSpStages * kSpTileBytes);
  unsigned char* qslot = ss_smem + kSsRingBytes + (size_t)warp * kSsSlots * 512;
  SsDesc* desc = reinterpret_cast<SsDesc*>(ss_smem + kSsRingBytes + kSsQBytes) + warp * kSsSlots;
  float* accbuf = reinterpret_cast<float*>(ss_smem + kSsRingBytes + kSsQBytes + kSsDescBytes) + warp * kHeadDim;
  const float scale = a.qv.sm_scale * kLog2e;
  const int qbytes = a.qv.q_f32 ? 512 : 256;
  uint32_t bad = 0;

  // ---- S3: task fetch and raw index loads.  The next task number is taken one task ahead.
  uint32_t tau_next = 0;
  if (lane == 0) tau_next = atomicAdd(a.sched, 1u);
  tau_next = __shfl_sync(FULL, tau_next, 0);
  int p_slot = 0, p_w = 0, p_nwin = 0, p_e0 = 0, p_e1 = 0;
  int64_t p_base = 0;
  uint32_t p_seq = 0;
  bool p_end = false;
  int32_t v3 = -1, prev3 = 0;
  float lw3 = 0.f;
  uint32_t tag3 = kTagBubble;

  auto produce = [&]() {
    const int32_t last_raw = __shfl_sync(FULL, v3, 31);
    if (!p_end && p_w + 1 < p_nwin) {   // the next window of the current task
      ++p_w;
      const int e = p_e0 + 32 * p_w + lane;
      v3 = e < p_e1 ? __ldg(a.idx + p_base + e) : -1;
      lw3 = (WEIGHTED && e < p_e1) ? __ldg(a.logw + p_base + e) * kLog2e : 0.f;
      prev3 = last_raw;
      tag3 = (uint32_t)p_slot | (p_w + 1 == p_nwin ? kTagLast : 0u);
      return;
    }
    for (;;) {   // the next task that has entries
      const int64_t tau = (int64_t)tau_next;
      if (p_end || tau >= total) {
        p_end = true;
        v3 = -1; prev3 = 0; lw3 = 0.f;
        tag3 = kTagEnd;
        return;
      }
      uint32_t nx = 0;
      if (lane == 0) nx = atomicAdd(a.sched, 1u);
      tau_next = __shfl_sync(FULL, nx, 0);
      // tasks are numbered chunk-major: (chunk, sequence, kv head, list).  Every list's chunk 0 is
      // handed out first, then every list's chunk 1, and so on, so all lists advance through
      // their entries together, as in a single wave: a row that several lists of a kv head
      // select (at similar ranks of their ascending lists) is read again while the first read is
      // still in L2.  Chunks past the end of short lists come last and are skipped at the fetch.
      const int64_t slots = (int64_t)a.kv.batch * a.kv.hkv * M;
      const int c = (int)(tau / slots);
      int64_t r = tau - (int64_t)c * slots;
      const int m = (int)(r % M);
      r /= M;
      const int g = (int)(r % a.kv.hkv);
      const int b = (int)(r / a.kv.hkv);
      const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, c == 0 && g == 0 && m == 0 && lane == 0);
      const int j = m / G;
      if (j >= si.n) continue;   // no list in this slot (fewer query tokens than the bound)
      const int list = (si.t0 + j) * a.qv.hq + g * G + (m - j * G);
      const int64_t base = (int64_t)list * a.k_max;
      const int e0 = c * E;
      const int e1 = min(e0 + E, a.k_max);
      const int e = e0 + lane;
      const int32_t v = e < e1 ? __ldg(a.idx + base + e) : -1;
      if (c > 0 && __shfl_sync(FULL, v, 0) == -1) continue;   // past the end of its list
      const int slot = (int)(p_seq++ % kSsSlots);
      if (lane == 0) {
        SsDesc d;
        d.list = list; d.c = c; d.e1 = e1; d.kvlen = kv_len_of(a.qv, si, j); d.b = b; d.g = g;
        d.pad0 = d.pad1 = 0;
        desc[slot] = d;
      }
      // the task's q row -> its slot; the copy joins the next tile's commit group, several groups
      // before the task's first tile is consumed
      if (lane * 16 < qbytes)
        cp_async16(qslot + slot * 512 + lane * 16, static_cast<const char*>(a.qv.q) + (int64_t)list * qbytes + lane * 16);
      __syncwarp();
      p_slot = slot; p_base = base; p_e0 = e0; p_e1 = e1; p_w = 0;
      p_nwin = (e1 - e0 + 31) >> 5;
      v3 = v;
      lw3 = (WEIGHTED && e < e1) ? __ldg(a.logw + base + e) * kLog2e : 0.f;
      prev3 = c > 0 ? __ldg(a.idx + base + e0 - 1) : 0;
      tag3 = (uint32_t)slot | kTagFirst | (p_nwin == 1 ? kTagLast : 0u);
      return;
    }
  };

  // ---- S2: a window's raw indices -> physical rows (checks as in the one-task kernel)
  auto resolve = [&](int32_t v, int32_t prev, uint32_t tag) -> uint32_t {
    uint32_t row = kInvalidRow;
    if (tag & (kTagBubble | kTagEnd)) return row;
    const SsDesc& d = desc[tag & kTagSlot];
    const int b = d.b, g = d.g, kvlen = d.kvlen;
    uint32_t before = __shfl_up_sync(FULL, (uint32_t)v, 1);
    if (lane == 0) before = (uint32_t)prev;
    if ((uint32_t)v < before) bad |= TSD_DEV_UNSORTED;
    if (v < -1 || v >= kvlen) bad |= TSD_DEV_BAD_INDEX;
    if (v >= 0 && v < kvlen) {
      row = kv_row(a.kv, b, g, v);
      if (row == kInvalidRow) bad |= TSD_DEV_BAD_PAGE;
    }
    return row;
  };

  // tile p (0 or 1) of a window whose rows are `rows` -> ring stage `stage` (an empty commit
  // group when the tile has no valid row)
  auto issue = [&](uint32_t rows, uint32_t vmask, int p, int stage) {
    if (((vmask >> (16 * p)) & 0xFFFFu) != 0u) {
      const uint32_t st = ring + (uint32_t)(stage * kSpTileBytes);
      const int cc = lane & 15;
#pragma unroll
      for (int i = 0; i < kSpTileRows / 2; ++i) {
        const int r = 2 * i + (lane >> 4);
        const uint32_t rr = __shfl_sync(FULL, rows, 16 * p + r);
        const bool ok = rr != kInvalidRow;
        const int64_t off = ok ? (int64_t)rr * kHeadDim : 0;
        const uint32_t so = sp_off(r, cc);
        cp_async16_zfill(st + so, reinterpret_cast<const uint4*>(a.kv.k + off) + cc, ok);
        cp_async16_zfill(st + kSpHalfBytes + so, reinterpret_cast<const uint4*>(a.kv.v + off) + cc, ok);
      }
    }
    cp_async_commit();
  };

  // ---- pipeline fill: S3 -> S2 -> S1 -> S0
  uint32_t tag0 = kTagBubble, tag1 = kTagBubble, tag2 = kTagBubble;
  uint32_t row1 = kInvalidRow, row2 = kInvalidRow;
  uint32_t vm0 = 0, vm1 = 0, vm2 = 0;
  float lw0 = 0.f, lw1 = 0.f, lw2 = 0.f;
  // one step: S0 <- S1 <- S2 <- resolve(S3) <- produce()
  auto shift = [&]() {
    tag0 = tag1; vm0 = vm1; lw0 = lw1;
    tag1 = tag2; row1 = row2; vm1 = vm2; lw1 = lw2;
    if (!(tag3 & (kTagBubble | kTagEnd | kTagFirst)) && __ballot_sync(FULL, v3 != -1) == 0u) {
      // a later window with no entries: its task ended with the window now in S1
      tag1 |= kTagLast;
      p_nwin = p_w;
      tag2 = kTagBubble; row2 = kInvalidRow; vm2 = 0u; lw2 = 0.f;
    } else {
      row2 = resolve(v3, prev3, tag3);
      vm2 = __ballot_sync(FULL, row2 != kInvalidRow);
      tag2 = tag3;
      lw2 = lw3;
    }
    produce();
  };
  // after the first window is produced and shifted twice it is in S1: its two tiles go into
  // stages 0 and 1, and one more shift makes it S0
  produce();
  shift();
  shift();
  issue(row1, vm1, 0, 0);
  issue(row1, vm1, 1, 1);
  shift();

  float m_run = -CUDART_INF_F, l_run = 0.f;
  float o[8][4];
  uint32_t qb[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    qb[i][0] = qb[i][1] = 0u;
  }
  int stage = 0;
  while (!(tag0 & kTagEnd)) {
    const bool real = !(tag0 & kTagBubble);
    int32_t nf = -1;   // first entry after the task's chunk (its list's end when -1)
    if (real && (tag0 & kTagFirst)) {
      // a new task: reset the state and read q from its slot.  The q copy was issued when the
      // window was produced, before its tiles: it is in the group of the window's first tile or
      // an older one, so all groups but the newest (the window's second tile) must be complete.
      m_run = -CUDART_INF_F;
      l_run = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      cp_async_wait<1>();
      __syncwarp();
      const int col = lane >> 2, i2 = 2 * (lane & 3);
      const unsigned char* qs = qslot + (tag0 & kTagSlot) * 512;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qb[ks][0] = qb[ks][1] = 0u;
        if (col < 2) {
          const int d0 = 16 * ks + i2;
          float x0, x1, y0, y1;
          if (a.qv.q_f32) {
            const float2 u = *reinterpret_cast<const float2*>(qs + 4 * d0);
            const float2 v = *reinterpret_cast<const float2*>(qs + 4 * (d0 + 8));
            x0 = u.x; x1 = u.y; y0 = v.x; y1 = v.y;
          } else {
            const uint32_t u = *reinterpret_cast<const uint32_t*>(qs + 2 * d0);
            const uint32_t v = *reinterpret_cast<const uint32_t*>(qs + 2 * (d0 + 8));
            x0 = bf16lo(u); x1 = bf16hi(u); y0 = bf16lo(v); y1 = bf16hi(v);
          }
          uint32_t h0, l0, h1, l1;
          split_bf16(x0, x1, h0, l0);
          split_bf16(y0, y1, h1, l1);
          qb[ks][0] = col == 0 ? h0 : l0;
          qb[ks][1] = col == 0 ? h1 : l1;
        }
      }
    }
    if (real && (tag0 & kTagLast)) {
      const SsDesc& d = desc[tag0 & kTagSlot];
      if (d.e1 < a.k_max) nf = __ldg(a.idx + (int64_t)d.list * a.k_max + d.e1);
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      // the same tile of the next window (S1) goes into the stage consumed last
      __syncwarp();
      issue(row1, vm1, p, stage == 0 ? kSpStages - 1 : stage - 1);
      cp_async_wait<kSpStages - 1>();
      __syncwarp();
      const uint32_t tmask = (vm0 >> (16 * p)) & 0xFFFFu;
      if (tmask != 0u)
        sp_tile<WEIGHTED>(ring + (uint32_t)(stage * kSpTileBytes), tmask, qb, scale, lw0, p, m_run, l_run, o);
      stage = stage + 1 == kSpStages ? 0 : stage + 1;
    }
    if (real && (tag0 & kTagLast)) {
      // finish the task: the lane sums of l, the O^T fragments -> 4 dims per lane
      const SsDesc d = desc[tag0 & kTagSlot];
      float l = l_run;
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) l += __shfl_xor_sync(FULL, l, o2);
      l = __shfl_sync(FULL, l, 0);
      if ((lane & 3) == 0) {
        const int i = lane >> 2;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          accbuf[16 * k + i] = o[k][0] + o[k][1];
          accbuf[16 * k + i + 8] = o[k][2] + o[k][3];
        }
      }
      __syncwarp();
      const float4 acc = *reinterpret_cast<const float4*>(accbuf + 4 * lane);
      __syncwarp();
      const int64_t list_id = d.list;
      const bool last_chunk = d.e1 >= a.k_max || __shfl_sync(FULL, nf, 0) == -1;
      if (C == 1 || (d.c == 0 && last_chunk)) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int t = d.list / a.qv.hq, h = d.list % a.qv.hq;
        store_out4(a, t, h, 4 * lane, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
        if (lane == 0 && a.lse != nullptr) a.lse[list_id] = l > 0.f ? (m_run + log2f(l)) * kLn2 : -CUDART_INF_F;
      } else {
        const int64_t pidx = list_id * a.nsplit + d.c;
        if (lane == 0) a.part_ml[pidx] = make_float2(l > 0.f ? m_run : -CUDART_INF_F, l);
        reinterpret_cast<float4*>(a.part_acc + pidx * kHeadDim)[lane] = acc;
        __threadfence();
        __syncwarp();
        uint32_t now = 0;
        if (lane == 0) {
          const uint32_t add = 1u + (last_chunk ? ((uint32_t)(d.c + 1) << 16) : 0u);
          now = atomicAdd(a.counters + list_id, add) + add;
        }
        now = __shfl_sync(FULL, now, 0);
        const uint32_t need = now >> 16;
        if (need != 0u && (now & 0xFFFFu) == need) {   // this arrival completed the list
          __threadfence();
          // a malformed list (entries after its -1 padding) can claim more chunks than it has:
          // the merge never reads past the list's own C partials
          merge_partials_of_list(a, list_id, (int)min(need, (uint32_t)C), lane);
          if (lane == 0) atomicExch(a.counters + list_id, 0u);
        }
      }
    }
    shift();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) bad |= __shfl_xor_sync(FULL, bad, o2);
  if (lane == 0 && bad) flag_status(a.status, bad);

  // the last warp of the grid to finish leaves the counters zero for the next call
  uint32_t done = 0;
  if (lane == 0) {
    __threadfence();
    done = atomicAdd(a.sched + 1, 1u);
  }
  done = __shfl_sync(FULL, done, 0);
  if (done + 1 == gridDim.x * (uint32_t)kSsWarps) {
    __threadfence();
    const int64_t lists = (int64_t)a.qv.num_tokens * a.qv.hq;
    for (int64_t i = lane; i < lists; i += 32) a.counters[i] = 0u;
    if (lane == 0) {
      a.sched[0] = 0u;
      a.sched[1] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// Dense decode on tensor cores
// ---------------------------------------------------------------------------
// One CTA per (sequence b, kv head g, list group lg, window of W tokens): up to 16 lists
// (q heads of the GQA group x decode tokens) are the rows of the mma M dimension.  A
// producer warp streams 64-token K/V tiles through a 2-stage ring (TMA, see tsd_kvtile.cuh);
// each of the 4 consumer warps takes 16 tokens of every tile:
//   S = q K^T (16 x 16, 8 k-steps of mma.m16n8k16), scaled to base-2 softmax units in fp32,
//   masked past each list's kv_len; online softmax per query row (quad shuffles);
//   O += P V with P split into bf16 hi + lo (two MMAs, ~16-bit weights) and V read with
//   transposing ldmatrix.
// The 4 warp states of each list are combined at the end and merged across windows like the
// sparse path's CTA partials.
constexpr int kDnStages = 2;
constexpr int kDnConsumers = 4;
constexpr int kDnThreads = 32 * (kDnConsumers + 1);
constexpr int kDnStageBytes = 2 * kTileBytesKV;   // K then V

struct DenseSmem {
  alignas(1024) unsigned char stage[kDnStages][kDnStageBytes];   // also the combine buffer
  alignas(1024) unsigned char qhi[kQTileBytes];
  alignas(1024) unsigned char qlo[kQTileBytes];
  uint64_t full[kDnStages];
  uint64_t empty[kDnStages];
  uint32_t abort;
  float mx[16], lsum[16];
};
static_assert(kDnStages * kDnStageBytes >= 16 * kDnConsumers * kCombFloats * 4, "dense combine buffer");
static_assert(sizeof(DenseSmem) + 1024 <= 75 * 1024, "three dense CTAs per SM");

template <bool QF32>
__global__ void __launch_bounds__(kDnThreads, kDnCtasPerSm) dense_decode_kernel(DecodeArgs a, const __grid_constant__ KvMaps maps) {
  extern __shared__ __align__(1024) unsigned char smem_dn[];
  DenseSmem& S = *reinterpret_cast<DenseSmem*>(smem_dn);
  const int split = blockIdx.x;
  const int g = blockIdx.y / a.list_groups, lg = blockIdx.y % a.list_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, split == 0 && g == 0 && lg == 0 && threadIdx.x == 0);
  const int G = a.qv.hq / a.kv.hkv;
  int nlists = si.n * G - lg * a.lists_per_cta;
  if (nlists > a.lists_per_cta) nlists = a.lists_per_cta;
  if (nlists <= 0) return;
  const int tok0 = split * a.span;
  const int tok_end = min(tok0 + a.span, si.len);
  const int ntiles = tok_end > tok0 ? (tok_end - tok0 + kTileTok - 1) / kTileTok : 0;
  const bool use_tma = a.kv.page_table == nullptr || a.kv.page_shift >= 3;
  // the swizzled tiles need 1024-byte alignment; refuse to run rather than mis-address them
  if (smem_u32(S.stage[0]) & 1023u) {
    if (threadIdx.x == 0) flag_status(a.status, TSD_DEV_TIMEOUT);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDnStages; ++s) {
      mbar_init(&S.full[s], use_tma ? 1 : 32);
      mbar_init(&S.empty[s], kDnConsumers);
    }
    mbar_fence_init();
    S.abort = 0;
  }
  store_q_tile(a.qv, si, g, G, lg * a.lists_per_cta, nlists, S.qhi, QF32 ? S.qlo : nullptr, threadIdx.x, kDnThreads);
  __syncthreads();

  // per warp state: rows r0 = lane/4 and r0 + 8
  float o[16][4];
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};

  if (warp == kDnConsumers) {
    produce_tiles<kDnStages, kDnStageBytes, true>(a.kv, maps, b, g, tok0, tok_end, ntiles, &S.stage[0][0], S.full,
                                                  S.empty, &S.abort, use_tma, lane, a.status);
  } else {
    const int w = warp;
    const float scale2 = a.qv.sm_scale * kLog2e;
    int kvl[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = (lane >> 2) + 8 * hr;
      kvl[hr] = m < nlists ? kv_len_of(a.qv, si, (lg * a.lists_per_cta + m) / G) : 0;
    }
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    const int i4 = lane >> 3, rr = lane & 7;
    for (int tile = 0; tile < ntiles; ++tile) {
      const int s = tile % kDnStages;
      if (!consume_wait<kDnStages>(S.full, &S.abort, tile, lane, a.status)) break;
      const unsigned char* kt = S.stage[s];
      const unsigned char* vt = S.stage[s] + kTileBytesKV;
      float sc[2][4];
      qk_tile<QF32>(S.qhi, S.qlo, kt, w, lane, sc);
      // scale, mask, online softmax per query row
      const int tbase = tok0 + tile * kTileTok + 16 * w + 2 * (lane & 3);
      float p[2][4];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float mloc = -CUDART_INF_F;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int tk = tbase + 8 * nt + j;
            float v = sc[nt][2 * hr + j] * scale2;
            if (tk >= kvl[hr] || tk >= tok_end) v = -CUDART_INF_F;
            sc[nt][2 * hr + j] = v;
            mloc = fmaxf(mloc, v);
          }
        mloc = fmaxf(mloc, __shfl_xor_sync(0xFFFFFFFFu, mloc, 1));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xFFFFFFFFu, mloc, 2));
        const float mnew = fmaxf(m_run[hr], mloc);
        const float alpha = mnew == -CUDART_INF_F ? 1.f : fast_exp2(m_run[hr] - mnew);
        float ps = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float v = sc[nt][2 * hr + j];
            const float pv = v == -CUDART_INF_F ? 0.f : fast_exp2(v - mnew);
            p[nt][2 * hr + j] = pv;
            ps += pv;
          }
        l_run[hr] = l_run[hr] * alpha + ps;
        m_run[hr] = mnew;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
          o[nd][2 * hr] *= alpha;
          o[nd][2 * hr + 1] *= alpha;
        }
      }
      // V rows of this warp's slice past the window end are stale shared memory or cache
      // slots beyond the sequence (possibly non-finite): zero them so that 0 * V stays 0
      const int slice0 = tok0 + tile * kTileTok + 16 * w;
      const bool zeroed = slice0 + 16 > tok_end;
      if (zeroed) {
        unsigned char* vw = S.stage[s] + kTileBytesKV;
        for (int i = lane; i < 16 * 16; i += 32) {   // 16 rows x (2 halves x 8 chunks of 16 B)
          const int r = i >> 4, hc = i & 15;
          if (slice0 + r >= tok_end)
            *reinterpret_cast<uint4*>(vw + (hc >> 3) * kHalfBytes + sw128(16 * w + r, hc & 7)) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // P (16 x 16) as the A operand: hi and lo bf16 parts
      uint32_t ph[4], pl[4];
      split_bf16(p[0][0], p[0][1], ph[0], pl[0]);
      split_bf16(p[0][2], p[0][3], ph[1], pl[1]);
      split_bf16(p[1][0], p[1][1], ph[2], pl[2]);
      split_bf16(p[1][2], p[1][3], ph[3], pl[3]);
      const uint32_t vbase = smem_u32(vt);
      const int tokrow = 16 * w + ((i4 & 1) << 3) + rr;
#pragma unroll
      for (int nd = 0; nd < 16; nd += 2) {
        const int dc = nd + (i4 >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + (dc >> 3) * kHalfBytes + sw128(tokrow, dc & 7), b0, b1, b2, b3);
        mma_bf16(o[nd], ph, b0, b1);
        mma_bf16(o[nd], pl, b0, b1);
        mma_bf16(o[nd + 1], ph, b2, b3);
        mma_bf16(o[nd + 1], pl, b2, b3);
      }
      __syncwarp();
      // order this warp's generic-proxy writes before the stage's next TMA refill
      if (zeroed) asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      if (lane == 0) mbar_arrive(&S.empty[s]);
    }
    // row sums over the quad
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      l_run[hr] += __shfl_xor_sync(0xFFFFFFFFu, l_run[hr], 1);
      l_run[hr] += __shfl_xor_sync(0xFFFFFFFFu, l_run[hr], 2);
    }
  }
  __syncthreads();
  // combine buffer: entry (list m, part = warp)
  float* comb = reinterpret_cast<float*>(S.stage[0]);
  if (warp < kDnConsumers) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = (lane >> 2) + 8 * hr;
      if (m < nlists) {
        float* e = comb + (size_t)(m * kDnConsumers + warp) * kCombFloats;
        if ((lane & 3) == 0) {
          e[0] = m_run[hr];
          e[1] = l_run[hr];
        }
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
          const int d = nd * 8 + 2 * (lane & 3);
          e[4 + d] = o[nd][2 * hr];
          e[4 + d + 1] = o[nd][2 * hr + 1];
        }
      }
    }
  }
  __syncthreads();
  finish_lists(a, si, b, g, lg, split, nlists, kDnConsumers, comb, S.mx, S.lsum);
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// The persistent form: kSsCtasPerSm CTAs per SM (fewer when there are fewer tasks).
static cudaError_t launch_sparse_stream(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream,
                                        bool dependent) {
  const int64_t tasks = (int64_t)batch * hkv * a.nsplit * a.lists_per_cta;
  if (tasks >= ((int64_t)1 << 31) || a.sched == nullptr) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int64_t grid = (int64_t)sms * kSsCtasPerSm;
  const int64_t need = (tasks + kSsWarps - 1) / kSsWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  static bool configured = false;
  if (!configured) {
    e = cudaFuncSetAttribute(sparse_stream_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSsSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(sparse_stream_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSsSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  auto kernel = a.logw != nullptr ? sparse_stream_kernel<true> : sparse_stream_kernel<false>;
  if (dependent) return launch_dependent(kernel, dim3((unsigned)grid), dim3(kSsThreads), kSsSmemBytes, stream, a);
  kernel<<<(unsigned)grid, kSsThreads, kSsSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream, bool dependent) {
  if (a.persistent) return launch_sparse_stream(a, batch, hkv, stream, dependent);
  const int64_t tasks = (int64_t)batch * hkv * a.nsplit * a.lists_per_cta;
  const int64_t grid = (tasks + kSpWarps - 1) / kSpWarps;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSpSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(sparse_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSpSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  auto kernel = a.logw != nullptr ? sparse_decode_kernel<true> : sparse_decode_kernel<false>;
  if (dependent) return launch_dependent(kernel, dim3((unsigned)grid), dim3(kSpThreads), kSpSmemBytes, stream, a);
  kernel<<<(unsigned)grid, kSpThreads, kSpSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dense_decode(const DecodeArgs& a, const KvMaps& maps, int batch, int hkv, cudaStream_t stream) {
  const size_t smem = sizeof(DenseSmem);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(dense_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dense_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(a.nsplit, hkv * a.list_groups, batch);
  if (a.qv.q_f32) {
    dense_decode_kernel<true><<<grid, kDnThreads, smem, stream>>>(a, maps);
  } else {
    dense_decode_kernel<false><<<grid, kDnThreads, smem, stream>>>(a, maps);
  }
  return cudaGetLastError();
}

}  // namespace tsd
