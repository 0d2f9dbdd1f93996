// Context-parallel (sequence-sharded) pieces of the decode step.
//
// With the KV cache of every sequence split over P ranks by token range (rank r's range
// before rank r + 1's), each rank runs the exact top-k on its shard and keeps its k best
// (score, shard-local token) candidates.  The global top-k is contained in the union of the
// P local top-k lists, so after the candidates are exchanged every rank re-selects the
// global top-k among the P x k candidates
// (cp_merge_select_kernel) and keeps the ones in its own shard.  Each rank then decodes
// over those rows and the P partial results (normalised output, log-sum-exp) are merged
// (merge_partials_kernel).  The exchange itself is not here: the candidates and partials
// are plain device arrays that the caller gathers rank-major, P x [lists][...].
//
// Candidate order: rank r's candidates all lie in its token range, which precedes rank
// r + 1's, and each rank's list is ascending, so the rank-major concatenation is ascending
// in the global token index without ever forming that index.  The select therefore keeps
// ties to the lower index by taking equal keys in array order -- the same rule as the
// single-GPU top-k.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "tsd_common.cuh"

namespace tsd {

constexpr int kCpThreads = 256;
constexpr int kCpMaxCand = 16384;   // P x k candidates per list held in shared memory
constexpr int kCpBins = 2048;

struct CpSmem {
  uint32_t key[kCpMaxCand];
  uint32_t hist[kCpBins];
  int scan_tmp[kCpThreads / 32 + 1];
  int found_bin, found_above;
};

__device__ void cp_find_bin(CpSmem& S, int nbins, int need) {
  if (threadIdx.x == 0) {
    S.found_bin = 0;
    S.found_above = 0;
  }
  const int per = (nbins + kCpThreads - 1) / kCpThreads;
  const int hi = nbins - threadIdx.x * per;
  int local = 0;
  for (int j = 0; j < per; ++j) {
    const int bin = hi - 1 - j;
    if (bin >= 0) local += (int)S.hist[bin];
  }
  int total;
  int run = block_exclusive_scan<kCpThreads>(local, S.scan_tmp, &total);
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

// One CTA per list.  cand_idx / cand_score: [P][lists][kc], each rank's shard-local token
// indices (-1 padding) and their scores.  Keeps the global top-k of the list (k =
// k_per_list[list] or k) and writes the kept candidates of rank my_rank (its local indices),
// ascending, -1 padded to k_out.
__global__ void __launch_bounds__(kCpThreads) cp_merge_select_kernel(const int32_t* cand_idx, const float* cand_score,
                                                                     int P, int64_t lists, int kc,
                                                                     const int32_t* k_per_list, int k_fixed,
                                                                     int my_rank, int32_t* out, int k_out,
                                                                     uint32_t* status) {
  extern __shared__ __align__(16) unsigned char cp_smem[];
  CpSmem& S = *reinterpret_cast<CpSmem*>(cp_smem);
  const int64_t list = blockIdx.x;
  const int n = P * kc;
  int k = k_per_list != nullptr ? __ldg(k_per_list + list) : k_fixed;
  int32_t* o = out + list * k_out;
  // candidate c = (rank c / kc, slot c % kc); padding keys are 0, below every real score's key
  int valid = 0;
  for (int c = threadIdx.x; c < n; c += kCpThreads) {
    const int64_t at = ((int64_t)(c / kc) * lists + list) * kc + (c % kc);
    const int32_t gi = __ldg(cand_idx + at);
    S.key[c] = gi >= 0 ? score_key(__ldg(cand_score + at)) : 0u;
    valid += gi >= 0;
  }
  int nvalid;
  block_exclusive_scan<kCpThreads>(valid, S.scan_tmp, &nvalid);
  if (k > nvalid) k = nvalid;
  if (k < 0) k = 0;
  // exact k-th key among the candidates (3 radix rounds), and how many ties are kept
  uint32_t prefix = 0u;
  int need = k, shift = 32;
  if (k > 0) {
    while (shift > 0) {
      const int nb = shift >= 11 ? 11 : shift;
      shift -= nb;
      const bool first = shift + nb == 32;
      for (int i = threadIdx.x; i < (1 << nb); i += kCpThreads) S.hist[i] = 0u;
      __syncthreads();
      for (int c = threadIdx.x; c < n; c += kCpThreads) {
        const uint32_t key = S.key[c];
        if (key != 0u && (first || (key >> (shift + nb)) == prefix))
          atomicAdd(&S.hist[(key >> shift) & ((1u << nb) - 1u)], 1u);
      }
      __syncthreads();
      cp_find_bin(S, 1 << nb, need);
      prefix = (prefix << nb) | (uint32_t)S.found_bin;
      need -= S.found_above;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;
  const int need_eq = need;
  // ordered pass: candidates are ascending in the global index; keep the shard's selected ones
  constexpr int kPer = kCpMaxCand / kCpThreads;   // 64 candidates per thread, in order
  const int c0 = threadIdx.x * kPer;
  int neq = 0;
  for (int j = 0; j < kPer; ++j) neq += (k > 0 && c0 + j < n && S.key[c0 + j] != 0u && S.key[c0 + j] == T);
  int eq_total;
  int eq_run = block_exclusive_scan<kCpThreads>(neq, S.scan_tmp, &eq_total);
  int nmine = 0;
  for (int j = 0; j < kPer; ++j) {
    const int c = c0 + j;
    if (k == 0 || c >= n || S.key[c] == 0u) continue;
    bool sel = S.key[c] > T;
    if (S.key[c] == T) sel = eq_run++ < need_eq;
    nmine += sel && c / kc == my_rank;
  }
  int mine_total;
  int pos = block_exclusive_scan<kCpThreads>(nmine, S.scan_tmp, &mine_total);
  eq_run = eq_run - neq;   // replay the tie ranks of this thread's candidates
  for (int j = 0; j < kPer; ++j) {
    const int c = c0 + j;
    if (k == 0 || c >= n || S.key[c] == 0u) continue;
    bool sel = S.key[c] > T;
    if (S.key[c] == T) sel = eq_run++ < need_eq;
    if (sel && c / kc == my_rank) {
      if (pos < k_out) o[pos] = __ldg(cand_idx + ((int64_t)my_rank * lists + list) * kc + (c % kc));
      else if (status != nullptr) flag_status(status, TSD_DEV_BAD_INDEX);
      ++pos;
    }
  }
  for (int i = mine_total + threadIdx.x; i < k_out; i += kCpThreads) o[i] = -1;
}

// One warp per row: out = sum_r w_r out_r / sum_r w_r, w_r = exp(lse_r - max lse), and
// lse = max + ln sum_r w_r; rows whose parts are all empty get out = 0, lse = -inf.
__global__ void merge_partials_kernel(int P, int64_t rows, const float* out_parts, const float* lse_parts, void* out,
                                      int out_f32, float* lse) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float mx = -CUDART_INF_F;
  for (int r = 0; r < P; ++r) mx = fmaxf(mx, __ldg(lse_parts + (int64_t)r * rows + row));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (mx != -CUDART_INF_F) {
    for (int r = 0; r < P; ++r) {
      const float l = __ldg(lse_parts + (int64_t)r * rows + row);
      const float w = l == -CUDART_INF_F ? 0.f : expf(l - mx);
      const float4 x = __ldg(reinterpret_cast<const float4*>(out_parts + ((int64_t)r * rows + row) * kHeadDim) + lane);
      acc.x = fmaf(w, x.x, acc.x); acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z); acc.w = fmaf(w, x.w, acc.w);
      den += w;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const float v[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  if (out_f32) {
    *(reinterpret_cast<float4*>(out) + row * 32 + lane) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    uint16_t* o = reinterpret_cast<uint16_t*>(out) + row * kHeadDim + 4 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = f32_to_bf16_rne(v[i]);
  }
  if (lane == 0 && lse != nullptr) lse[row] = den > 0.f ? mx + logf(den) : -CUDART_INF_F;
}

cudaError_t launch_cp_merge_select(const int32_t* cand_idx, const float* cand_score, int P, int64_t lists, int kc,
                                   const int32_t* k_per_list, int k, int my_rank, int32_t* out, int k_out,
                                   uint32_t* status, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(cp_merge_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(CpSmem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (lists > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  cp_merge_select_kernel<<<(unsigned)lists, kCpThreads, sizeof(CpSmem), stream>>>(
      cand_idx, cand_score, P, lists, kc, k_per_list, k, my_rank, out, k_out, status);
  return cudaGetLastError();
}

int cp_max_candidates() { return kCpMaxCand; }

cudaError_t launch_merge_partials(int P, int64_t rows, const float* out_parts, const float* lse_parts, void* out,
                                  int out_f32, float* lse, cudaStream_t stream) {
  const int64_t blocks = (rows * 32 + 255) / 256;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  merge_partials_kernel<<<(unsigned)blocks, 256, 0, stream>>>(P, rows, out_parts, lse_parts, out, out_f32, lse);
  return cudaGetLastError();
}

}  // namespace tsd
