// Sparse and dense decode attention kernels for sm_100a.
//
// Operation ("Inference Time Context Sparsity: Illusion or Opportunity?",
// gist.science summary, section 2 "Hardware implementation" and section 3.C):
// for each (query token t, q head h) attend only to the K/V rows named by its
// index list -- which may differ per token, per query and per head -- so that
// the bytes read fall from O(N d) to O(k d).  Dense decode attends to every row.
//
// Sparse decode: one half-warp per task (16+ entries of one list); rows gathered through a
// per-half-warp cp.async ring; batched online softmax; per-list split-K merge in the CTA,
// then by the last CTA of the list to finish.
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
//  * Scattered 256-byte rows are gathered with 16-byte copies: lane l of a half-warp copies
//    chunk l of each K and V row.  The copies go through a per-half-warp ring of kSpStages
//    batches in shared memory (cp.async), so 12 rows are in flight per half-warp without
//    spending registers on them.  Each lane reads back only what it copied itself, so the
//    ring needs no synchronisation beyond each lane's own cp.async wait.  Against gathering
//    into registers (4 rows in flight, 3 CTAs/SM) this measured 30.7 vs 32.8 us on
//    llama3_8b.
//  * What sets the gather rate is how many loads are in flight, so the work is cut into many
//    small independent tasks: one half-warp (16 lanes x 16 bytes = one row) takes a chunk of
//    E entries of one list (token x q head) and nothing else, and the plan sizes E so the
//    grid fits one wave of resident CTAs.
//  * Tasks are numbered (sequence, kv head, chunk, list) so that the lists of one kv head
//    -- the q heads of a GQA group and the decode tokens of the sequence -- read the same
//    token range in the same CTA at the same time: a row picked by several of them is
//    read from DRAM once and served to the others from L2.
// Per row the half-warp computes a 128-dim dot (8 FMA per lane + a 4-step shuffle
// reduction); its online softmax state (max, sum, 8 output dims per lane) is updated once
// per batch of U rows.  The chunks of a list held by one CTA are combined in shared memory;
// each CTA then writes one partial per list, and the last CTA of a list to arrive (a per-list
// counter) merges them with log-sum-exp.  A list that fits one CTA is written directly.
constexpr int kSpThreads = 256;   // 16 half-warps, one task each
constexpr int kSpU = 4;           // rows per softmax batch
constexpr int kSpStages = 3;      // batches in flight per half-warp (cp.async ring)
constexpr size_t kSpRingBytes = (size_t)16 * kSpStages * 2 * kSpU * 16 * sizeof(uint4);   // 96 KB

__device__ __forceinline__ void row_fetch(const DecodeArgs& a, uint32_t row, int l, uint4& k, uint4& v) {
  if (row != kInvalidRow) {
    k = __ldg(reinterpret_cast<const uint4*>(a.kv.k + (int64_t)row * kHeadDim) + l);
    v = __ldg(reinterpret_cast<const uint4*>(a.kv.v + (int64_t)row * kHeadDim) + l);
  }
}

// Online-softmax update of a half-warp's state with a batch of U rows at once: the U
// scores are reduced together (independent shuffle chains), then one max, one rescale
// and U independent exponentials -- the serial chain is per batch, not per row.
template <int U, bool BIAS>
__device__ __forceinline__ void batch_update(const uint4* kq, const uint4* vq, const uint32_t* rr, const float* bias,
                                             const float* q, float& m_run, float& l_run, float* acc, unsigned hmask) {
  float s[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float kf[8];
    unpack8(kq[u], kf);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      s0 = fmaf(q[j], kf[j], s0);
      s1 = fmaf(q[j + 1], kf[j + 1], s1);
    }
    s[u] = s0 + s1;
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1)
#pragma unroll
    for (int u = 0; u < U; ++u) s[u] += __shfl_xor_sync(hmask, s[u], o);
  if (BIAS) {   // entry weights: p_i = w_i exp(s_i), with ln w_i in base-2 units
#pragma unroll
    for (int u = 0; u < U; ++u) s[u] += bias[u];
  }
  float mb = -CUDART_INF_F;
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (rr[u] != kInvalidRow) mb = fmaxf(mb, s[u]);
  if (mb == -CUDART_INF_F) return;   // no valid row in the batch (uniform over the half-warp)
  const float m_new = fmaxf(m_run, mb);
  const float alpha = fast_exp2(m_run - m_new);   // 0 on the first batch (m_run = -inf)
  l_run *= alpha;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] *= alpha;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const float p = rr[u] != kInvalidRow ? fast_exp2(s[u] - m_new) : 0.f;
    l_run += p;
    float vf[8];
    unpack8(vq[u], vf);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = fmaf(p, vf[j], acc[j]);
  }
  m_run = m_new;
}

// End of a list's work in one CTA: a list whose tasks all ran in this CTA is written
// directly; otherwise this CTA's partial state (partial c of C) is stored, and the last CTA
// of the list to arrive (per-list counter) merges the C partials with log-sum-exp.  Called
// by the 16 lanes of one half-warp (hmask), lane l holding output dims [8l, 8l+8).
__device__ __forceinline__ void finish_task(const DecodeArgs& a, int64_t list_id, int t, int h, int C, int c,
                                            float m_run, float l_run, const float* acc, int l, unsigned hmask) {
  if (C == 1) {   // the whole list in one CTA
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) store_out(a, t, h, 8 * l + i, acc[i] * inv);
    if (l == 0 && a.lse != nullptr) a.lse[list_id] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -CUDART_INF_F;
    return;
  }
  // partial of this task, then the per-list arrival count
  const int64_t pidx = list_id * a.nsplit + c;
  if (l == 0) a.part_ml[pidx] = make_float2(m_run, l_run);
  float4* pa = reinterpret_cast<float4*>(a.part_acc + pidx * kHeadDim + 8 * l);
  pa[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  pa[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  __threadfence();
  __syncwarp(hmask);
  uint32_t prev = 0;
  if (l == 0) {
    prev = atomicAdd(a.counters + list_id, 1u);
    if (prev == (uint32_t)(C - 1)) atomicExch(a.counters + list_id, 0u);   // leave it zero for the next call
  }
  prev = __shfl_sync(hmask, prev, 0, 16);
  if (prev != (uint32_t)(C - 1)) return;
  __threadfence();
  // last task of the list: merge its C partials (lanes over splits for the max and sum,
  // then 8 output dims per lane with independent loads)
  const float2* ml = a.part_ml + list_id * a.nsplit;
  float mx = -CUDART_INF_F;
  for (int i = l; i < C; i += 16) mx = fmaxf(mx, __ldcg(&ml[i]).x);
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 2));
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 4));
  mx = fmaxf(mx, __shfl_xor_sync(hmask, mx, 8));
  float L = 0.f;
  float o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  if (mx != -CUDART_INF_F) {
    for (int i = l; i < C; i += 16) {
      const float2 x = __ldcg(&ml[i]);
      L = fmaf(fast_exp2(x.x - mx), x.y, L);
    }
    L += __shfl_xor_sync(hmask, L, 1);
    L += __shfl_xor_sync(hmask, L, 2);
    L += __shfl_xor_sync(hmask, L, 4);
    L += __shfl_xor_sync(hmask, L, 8);
    for (int c0 = 0; c0 < C; c0 += 4) {
      float w[4];
      float4 x0[4], x1[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int cc = c0 + u;
        w[u] = cc < C ? fast_exp2(__ldcg(&ml[cc]).x - mx) : 0.f;
        const float4* src =
            reinterpret_cast<const float4*>(a.part_acc + (list_id * a.nsplit + (cc < C ? cc : 0)) * kHeadDim + 8 * l);
        x0[u] = __ldcg(src);
        x1[u] = __ldcg(src + 1);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        o[0] = fmaf(w[u], x0[u].x, o[0]); o[1] = fmaf(w[u], x0[u].y, o[1]);
        o[2] = fmaf(w[u], x0[u].z, o[2]); o[3] = fmaf(w[u], x0[u].w, o[3]);
        o[4] = fmaf(w[u], x1[u].x, o[4]); o[5] = fmaf(w[u], x1[u].y, o[5]);
        o[6] = fmaf(w[u], x1[u].z, o[6]); o[7] = fmaf(w[u], x1[u].w, o[7]);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) store_out(a, t, h, 8 * l + i, o[i] * inv);
  if (l == 0 && a.lse != nullptr) a.lse[list_id] = L > 0.f ? (mx + log2f(L)) * kLn2 : -CUDART_INF_F;
}

template <bool WEIGHTED>
__global__ void __launch_bounds__(kSpThreads, kSpCtasPerSm) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) uint4 sp_ring[];   // [16 half-warps][kSpStages][K, V][kSpU rows][16 lanes]
  // task states of the CTA's 16 half-warps, combined per list before anything leaves the CTA
  __shared__ float2 s_ml[16];
  __shared__ __align__(16) float s_acc[16][kHeadDim];
  __shared__ int64_t s_list[16];
  const int lane = threadIdx.x & 31;
  const int l = threadIdx.x & 15;
  const int hw = threadIdx.x >> 4;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int G = a.qv.hq / a.kv.hkv;
  const int M = a.lists_per_cta;   // list slots per (sequence, kv head): G x max tokens per sequence
  const int C = a.nsplit;          // tasks (chunks) per list
  const int E = a.span;            // entries per task
  const int64_t task = (int64_t)blockIdx.x * 16 + hw;
  const int64_t total = (int64_t)a.kv.batch * a.kv.hkv * C * M;
  const int64_t tk = task < total ? task : total - 1;
  const int m = (int)(tk % M);
  int64_t rest = tk / M;
  const int c = (int)(rest % C);
  rest /= C;
  const int g = (int)(rest % a.kv.hkv);
  const int b = (int)(rest / a.kv.hkv);

  const SeqInfo si = seq_info(a.kv, a.qv, b, a.status, task == tk && c == 0 && g == 0 && m == 0 && l == 0);
  const int j = m / G;
  const bool valid = task < total && j < si.n;   // no list for slots past this sequence's tokens
  const int t = si.t0 + j, h = g * G + (m - j * G);
  const int64_t list_id = valid ? (int64_t)t * a.qv.hq + h : -1;
  float m_run = -CUDART_INF_F, l_run = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  if (valid) {
    const int kvlen = kv_len_of(a.qv, si, j);
    const float scale = a.qv.sm_scale * kLog2e;
    // this lane's 8 query dims [8l, 8l+8), scaled so that dots are base-2 softmax units
    float q[8];
    {
      const int64_t qb = list_id * kHeadDim + 8 * l;
      if (a.qv.q_f32) {
        const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.qv.q) + qb);
        const float4 x = __ldg(p), y = __ldg(p + 1);
        q[0] = x.x; q[1] = x.y; q[2] = x.z; q[3] = x.w; q[4] = y.x; q[5] = y.y; q[6] = y.z; q[7] = y.w;
      } else {
        unpack8(__ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.qv.q) + qb)), q);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] *= scale;
    }

    const int32_t* lst = a.idx + list_id * a.k_max;
    const int e0 = c * E;
    const int e1 = min(e0 + E, a.k_max);
    uint32_t bad = 0;
    for (int base = e0; base < e1; base += 16) {
      // this lane's entry: index, predecessor check, validity, physical row
      const int e = base + l;
      const int32_t v = e < e1 ? __ldg(lst + e) : -1;
      uint32_t before = __shfl_up_sync(hmask, (uint32_t)v, 1, 16);
      if (l == 0 && e > 0 && e < e1) before = (uint32_t)__ldg(lst + e - 1);
      if (e < e1 && e > 0 && (uint32_t)v < before) bad |= TSD_DEV_UNSORTED;
      if (e < e1 && (v < -1 || v >= kvlen)) bad |= TSD_DEV_BAD_INDEX;
      uint32_t row = kInvalidRow;
      if (e < e1 && v >= 0 && v < kvlen) {
        row = kv_row(a.kv, b, g, v);
        if (row == kInvalidRow) bad |= TSD_DEV_BAD_PAGE;
      }
      float lw = 0.f;
      if (WEIGHTED && e < e1) lw = __ldg(a.logw + list_id * a.k_max + e) * kLog2e;
      // the 16 rows, kSpU at a time, through this half-warp's ring of kSpStages stages in
      // shared memory (cp.async): lane l copies, and later reads, chunk l of every row, so the
      // ring needs no synchronisation beyond each lane's own cp.async wait
      uint4* ring = sp_ring + (size_t)hw * kSpStages * 2 * kSpU * 16;
      auto issue = [&](int bt) {
        uint4* st = ring + (size_t)(bt % kSpStages) * 2 * kSpU * 16;
#pragma unroll
        for (int u = 0; u < kSpU; ++u) {
          const uint32_t rr = __shfl_sync(hmask, row, bt * kSpU + u, 16);
          if (rr != kInvalidRow) {
            cp_async16(st + u * 16 + l, reinterpret_cast<const uint4*>(a.kv.k + (int64_t)rr * kHeadDim) + l);
            cp_async16(st + (kSpU + u) * 16 + l, reinterpret_cast<const uint4*>(a.kv.v + (int64_t)rr * kHeadDim) + l);
          }
        }
        cp_async_commit();
      };
#pragma unroll
      for (int bt = 0; bt < kSpStages - 1; ++bt) issue(bt);
#pragma unroll
      for (int bt = 0; bt < 16 / kSpU; ++bt) {
        if (bt + kSpStages - 1 < 16 / kSpU) issue(bt + kSpStages - 1); else cp_async_commit();
        cp_async_wait<kSpStages - 1>();
        const uint4* st = ring + (size_t)(bt % kSpStages) * 2 * kSpU * 16;
        uint32_t rr[kSpU];
        float bias[kSpU];
        uint4 kq[kSpU], vq[kSpU];
#pragma unroll
        for (int u = 0; u < kSpU; ++u) {
          rr[u] = __shfl_sync(hmask, row, bt * kSpU + u, 16);
          bias[u] = WEIGHTED ? __shfl_sync(hmask, lw, bt * kSpU + u, 16) : 0.f;
          kq[u] = rr[u] != kInvalidRow ? st[u * 16 + l] : make_uint4(0, 0, 0, 0);
          vq[u] = rr[u] != kInvalidRow ? st[(kSpU + u) * 16 + l] : make_uint4(0, 0, 0, 0);
        }
        batch_update<kSpU, WEIGHTED>(kq, vq, rr, bias, q, m_run, l_run, acc, hmask);
      }
    }
    bad |= __shfl_xor_sync(hmask, bad, 1);
    bad |= __shfl_xor_sync(hmask, bad, 2);
    bad |= __shfl_xor_sync(hmask, bad, 4);
    bad |= __shfl_xor_sync(hmask, bad, 8);
    if (l == 0 && bad) flag_status(a.status, bad);
  }

  if (C == 1) {   // every list is one task (uniform over the grid)
    if (valid) finish_task(a, list_id, t, h, 1, 0, m_run, l_run, acc, l, hmask);
    return;
  }
  // Chunks c, c+1, ... of a list are M tasks apart, so a CTA holds up to 16/M consecutive
  // chunks of each of its lists.  Their states are combined here, and each list leaves the
  // CTA as a single partial: the cross-CTA merge reads (16/M)x fewer partials.
  if (l == 0) {
    s_ml[hw] = make_float2(m_run, l_run);
    s_list[hw] = list_id;
  }
  *reinterpret_cast<float4*>(&s_acc[hw][8 * l]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  *reinterpret_cast<float4*>(&s_acc[hw][8 * l + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  __syncthreads();
  if (!valid || (hw >= M && s_list[hw - M] == list_id)) return;   // not the first chunk of its list here
  for (int o = hw + M; o < 16 && s_list[o] == list_id; o += M) {
    const float2 x = s_ml[o];
    const float mn = fmaxf(m_run, x.x);
    if (mn == -CUDART_INF_F) continue;
    const float wa = fast_exp2(m_run - mn), wb = fast_exp2(x.x - mn);
    l_run = l_run * wa + x.y * wb;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = acc[i] * wa + s_acc[o][8 * l + i] * wb;
    m_run = mn;
  }
  // partials of the list = CTAs that hold one of its chunks (with M <= 16 every CTA from the
  // first chunk's to the last chunk's holds one); this CTA's partial index
  int parts = C, part = c;
  if (M <= 16) {
    const int64_t first = (((int64_t)b * a.kv.hkv + g) * C) * M + m;
    const int64_t last = first + (int64_t)(C - 1) * M;
    parts = (int)((last >> 4) - (first >> 4) + 1);
    part = (int)((int64_t)blockIdx.x - (first >> 4));
  }
  finish_task(a, list_id, t, h, parts, part, m_run, l_run, acc, l, hmask);
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
cudaError_t launch_sparse_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream) {
  const int64_t tasks = (int64_t)batch * hkv * a.nsplit * a.lists_per_cta;
  const int64_t grid = (tasks + 15) / 16;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSpRingBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(sparse_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSpRingBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (a.logw != nullptr) {
    sparse_decode_kernel<true><<<(unsigned)grid, kSpThreads, kSpRingBytes, stream>>>(a);
  } else {
    sparse_decode_kernel<false><<<(unsigned)grid, kSpThreads, kSpRingBytes, stream>>>(a);
  }
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
