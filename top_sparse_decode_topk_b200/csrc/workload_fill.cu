// Device side of the seeded workload generator (libtsd_workload.so).
//
// Fills a bf16 K or V cache with the same values the host generator produces:
// element d of token i of (sequence b, kv head g) of tensor `tensor_id` is lane
// d % 8 of Philox4x32-10 (Salmon et al., SC 2011) with counter
// (i, d/8 + 16 g + 65536 b, tensor_id, 0) and key (seed_lo, seed_hi), mapped
// through a 65536-entry table of bf16 normal quantiles.  Only slots that hold a
// token (i < seq_lens[b]) are written; the rest keep what the caller put there.
// This is input generation, not part of the attention path.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox_round(uint32_t& c0, uint32_t& c1, uint32_t& c2, uint32_t& c3, uint32_t k0,
                                             uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
  const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
  const uint32_t n0 = hi1 ^ c1 ^ k0;
  const uint32_t n2 = hi0 ^ c3 ^ k1;
  c0 = n0;
  c1 = lo1;
  c2 = n2;
  c3 = lo0;
}

__global__ void fill_kv_kernel(uint16_t* out, const uint16_t* __restrict__ table, const int32_t* __restrict__ page_table,
                               const int32_t* __restrict__ seq_lens, int batch, int hkv, int page_shift, int max_pages,
                               int max_seq_len, uint32_t seed_lo, uint32_t seed_hi, uint32_t tensor_id) {
  // one thread per (b, g, token, 8-element block)
  const int64_t total = (int64_t)batch * hkv * max_seq_len * 16;
  for (int64_t id = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; id < total; id += (int64_t)gridDim.x * blockDim.x) {
    const int blk = (int)(id & 15);
    int64_t rest = id >> 4;
    const int i = (int)(rest % max_seq_len);
    rest /= max_seq_len;
    const int g = (int)(rest % hkv);
    const int b = (int)(rest / hkv);
    if (i >= seq_lens[b]) continue;
    uint32_t c0 = (uint32_t)i, c1 = (uint32_t)blk + 16u * (uint32_t)g + 65536u * (uint32_t)b, c2 = tensor_id, c3 = 0;
    uint32_t k0 = seed_lo, k1 = seed_hi;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      philox_round(c0, c1, c2, c3, k0, k1);
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t w[4] = {c0, c1, c2, c3};
    uint16_t v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = table[w[j] & 0xFFFFu];
      v[2 * j + 1] = table[w[j] >> 16];
    }
    int64_t row;
    if (page_table == nullptr) {
      row = ((int64_t)b * hkv + g) * max_seq_len + i;
    } else {
      const int page = page_table[(int64_t)b * max_pages + (i >> page_shift)];
      row = (((int64_t)page * hkv + g) << page_shift) | (i & ((1 << page_shift) - 1));
    }
    uint4 pk;
    pk.x = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
    pk.y = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
    pk.z = (uint32_t)v[4] | ((uint32_t)v[5] << 16);
    pk.w = (uint32_t)v[6] | ((uint32_t)v[7] << 16);
    *reinterpret_cast<uint4*>(out + row * 128 + blk * 8) = pk;
  }
}

}  // namespace

extern "C" int tsdw_fill_kv(void* out, const void* table, const void* page_table, const void* seq_lens, int batch,
                            int hkv, int page_size, int max_pages, int max_seq_len, uint32_t seed_lo, uint32_t seed_hi,
                            uint32_t tensor_id, void* stream) {
  int shift = 0;
  const bool contiguous = page_size == 0;   // 0 selects [batch][hkv][max_seq_len][128]
  if (!contiguous) {
    while ((1 << shift) < page_size) ++shift;
    if ((1 << shift) != page_size) return (int)cudaErrorInvalidValue;
  }
  const int threads = 256;
  const int blocks = 148 * 8;
  fill_kv_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t*>(out), static_cast<const uint16_t*>(table),
      contiguous ? nullptr : static_cast<const int32_t*>(page_table), static_cast<const int32_t*>(seq_lens), batch, hkv,
      shift, max_pages, max_seq_len, seed_lo, seed_hi, tensor_id);
  return (int)cudaGetLastError();
}
