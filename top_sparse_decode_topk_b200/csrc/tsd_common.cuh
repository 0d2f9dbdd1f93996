// Device-side helpers shared by the sm_100a kernels of libtsd.
//
// Storage: K and V are bf16 rows of 128 elements (256 bytes per (token, kv head)),
// either in HND pages [page][kv head][slot][128] or contiguous
// [sequence][kv head][token][128].  All arithmetic is fp32.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tsd_plan.h"

namespace tsd {

constexpr int kHeadDim = 128;
constexpr uint32_t kInvalidRow = 0xFFFFFFFFu;

// ---------------------------------------------------------------------------
// Views passed by value to the kernels
// ---------------------------------------------------------------------------
struct KvView {
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* page_table;  // nullptr for the contiguous layout
  const int32_t* seq_lens;
  int64_t num_pages;
  int32_t hkv;
  int32_t page_shift;         // log2(page_size) (paged)
  int32_t max_pages;          // page-table row stride (paged)
  int32_t max_seq_len;
  int32_t batch;
};

struct QView {
  const void* q;
  int32_t q_f32;              // 1: fp32 queries, 0: bf16
  int32_t hq;
  int32_t num_tokens;
  const int32_t* q_indptr;    // nullptr: token b belongs to sequence b
  int32_t max_tokens;         // host bound on tokens per sequence
  int32_t causal;
  float sm_scale;
};

// Physical row (units of 128 elements) of token i of (sequence b, kv head g), or
// kInvalidRow when its page id is out of range (the caller flags TSD_DEV_BAD_PAGE).
__device__ __forceinline__ uint32_t kv_row(const KvView& kv, int b, int g, int i) {
  if (kv.page_table == nullptr) {
    return (uint32_t)(((int64_t)b * kv.hkv + g) * kv.max_seq_len + i);
  }
  const int32_t page = __ldg(kv.page_table + (int64_t)b * kv.max_pages + (i >> kv.page_shift));
  if (page < 0 || (int64_t)page >= kv.num_pages) return kInvalidRow;
  const int32_t mask = (1 << kv.page_shift) - 1;
  return (uint32_t)((((int64_t)page * kv.hkv + g) << kv.page_shift) | (i & mask));
}

// Tokens [t0, t0 + n) of sequence b, validated against the host bounds.  A bad
// descriptor makes the sequence empty and raises TSD_DEV_BAD_SEQ.
struct SeqInfo {
  int t0;
  int n;        // query tokens of the sequence
  int len;      // cached tokens (seq_lens[b])
};

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  atomicOr(status, bits);
}

// The raw descriptor of sequence b (seq_lens[b] and its q_indptr range), loaded but not yet
// checked, so that a kernel can put other loads in flight before it waits on these.
struct SeqRaw {
  int len, t0, t1;
};

__device__ __forceinline__ SeqRaw seq_load(const KvView& kv, const QView& qv, int b) {
  SeqRaw r;
  r.len = __ldg(kv.seq_lens + b);
  if (qv.q_indptr != nullptr) {
    r.t0 = __ldg(qv.q_indptr + b);
    r.t1 = __ldg(qv.q_indptr + b + 1);
  } else {
    r.t0 = b;
    r.t1 = b + 1;
  }
  return r;
}

__device__ __forceinline__ SeqInfo seq_check(const KvView& kv, const QView& qv, const SeqRaw& r, uint32_t* status,
                                             bool report) {
  SeqInfo s;
  const bool bad = r.len < 0 || r.len > kv.max_seq_len || r.t0 < 0 || r.t1 < r.t0 || r.t1 > qv.num_tokens ||
                   (r.t1 - r.t0) > qv.max_tokens;
  if (bad) {
    if (report) flag_status(status, TSD_DEV_BAD_SEQ_BIT);
    s.t0 = 0; s.n = 0; s.len = 0;
    return s;
  }
  s.t0 = r.t0; s.n = r.t1 - r.t0; s.len = r.len;
  return s;
}

__device__ __forceinline__ SeqInfo seq_info(const KvView& kv, const QView& qv, int b, uint32_t* status,
                                            bool report) {
  return seq_check(kv, qv, seq_load(kv, qv, b), status, report);
}

// Tokens visible to query j (0-based) of the n tokens of a sequence with len cached tokens.
__device__ __forceinline__ int kv_len_of(const QView& qv, const SeqInfo& s, int j) {
  int L = qv.causal ? s.len - s.n + j + 1 : s.len;
  return L < 0 ? 0 : L;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (a kernel launched with the programmatic stream serialization
// attribute may start while the previous kernel of the stream drains)
// ---------------------------------------------------------------------------
// In the dependent kernel: wait until the previous kernel has completed and its writes are
// visible.  A no-op when the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// In the previous kernel: this CTA no longer holds back the dependent kernel's launch (which
// starts once every CTA has done so or exited; it still waits in pdl_wait for completion).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// Numerics
// ---------------------------------------------------------------------------
// 2^x via the hardware approximation (ex2.approx, documented PTX instruction).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes of one 64-bit register (Blackwell's packed fp32x2 arithmetic): d = a * b + c
// lane by lane, each lane rounded as a scalar fmaf.
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// A bf16 pair (low half = first element) -> the fp32 pair in one 64-bit register (exact).
__device__ __forceinline__ unsigned long long bf16x2_to_f32x2(uint32_t w) {
  return ((unsigned long long)(w & 0xFFFF0000u) << 32) | (unsigned long long)(w << 16);
}
__device__ __forceinline__ float f32x2_sum(unsigned long long v) {
  return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

// Two bf16 packed in a 32-bit word -> two fp32 (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x);
  f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z); f[5] = bf16hi(u.z);
  f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Order-preserving map of an fp32 score onto uint32 (larger score -> larger key);
// -0.0 is folded onto +0.0 so that equal scores tie on the index.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score of an order-preserving key (inverse of score_key; -0 comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// ---------------------------------------------------------------------------
// Asynchronous global->shared copies (cp.async, 16 bytes, L2-only caching)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Arrive on `bar` once all of this thread's earlier cp.async copies have landed (the
// barrier's expected arrival count must include this thread).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"((uint32_t)__cvta_generic_to_shared(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// mbarriers and bulk (TMA, 1-D) copies
// ---------------------------------------------------------------------------
// Every wait on an mbarrier is bounded: after kWaitCycles SM cycles (about a second) it
// gives up and the caller reports TSD_DEV_TIMEOUT instead of hanging.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// try_wait that may suspend the thread until the phase completes or about `ns` nanoseconds
// pass, instead of returning at once: a waiting warp then takes no issue slots from the others.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, 1000000u)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}
// Global -> shared bulk copy (16-byte aligned addresses, size a multiple of 16) that
// signals completion on `bar` (complete_tx of `bytes`).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Asynchronous prefetch of `bytes` (multiple of 16, 16-byte aligned) from global memory
// into L2; it holds no register or shared-memory resources while in flight.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------
// TMA tensor loads and warp-level bf16 tensor-core MMA
// ---------------------------------------------------------------------------
// L2 policy for streams that are read once (the K/V tiles of dense decode and top-k scoring):
// their lines are the first to be evicted, so the stream does not push out data that the next
// kernel reads from L2 (the score workspace between scoring and selection).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// 2-D tiled TMA load (box given by the tensor map) into shared memory under an L2 cache
// policy, completion counted on `bar`.  x is the innermost (element) coordinate and must be a
// multiple of 8 for bf16 (16 bytes); y is the row.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const void* tmap, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;\n" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// cp_async16 with an L2 cache policy.
__device__ __forceinline__ void cp_async16_hint(void* smem, const void* gmem, uint64_t policy) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "l"(policy)
               : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-row tile written by TMA
// with 128-byte swizzling (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D += A(16x16, bf16, row) * B(16x8, bf16, col), fp32 accumulate
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two fp32 -> packed bf16x2 (round to nearest even); lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  return (uint32_t)f32_to_bf16_rne(lo) | ((uint32_t)f32_to_bf16_rne(hi) << 16);
}
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): the pair carries ~16 significant bits.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const uint16_t h0 = f32_to_bf16_rne(x0), h1 = f32_to_bf16_rne(x1);
  hi = (uint32_t)h0 | ((uint32_t)h1 << 16);
  lo = pack_bf16(x0 - __uint_as_float((uint32_t)h0 << 16), x1 - __uint_as_float((uint32_t)h1 << 16));
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (blockDim.x == NT, multiple of 32)
// ---------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tmp /* >= NT/32 + 1 */, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) warp_tmp[lane] = w;   // inclusive prefix of warp totals
    if (lane == NT / 32 - 1) warp_tmp[NT / 32] = w;
  }
  __syncthreads();
  int excl = x - v + (warp > 0 ? warp_tmp[warp - 1] : 0);
  *total = warp_tmp[NT / 32];
  __syncthreads();
  return excl;
}

// Launch `kernel` on `stream` as a programmatic dependent of the kernel before it: it may start
// while that kernel drains, and must call pdl_wait() before it reads anything that kernel writes.
template <typename... Args>
cudaError_t launch_dependent(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace tsd
