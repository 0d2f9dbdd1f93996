// Sparse decode without a caller-supplied workspace.
//
// Some callers cannot allocate device memory for the workspace: a plugin that
// runs inside another runtime which owns every device allocation, or a decode
// loop that must not call cudaMalloc (it synchronizes the whole device) and has
// no way to thread a workspace pointer down to this call.  For them,
// tsd_sparse_decode_static_ws runs the same sparse decode kernel as
// tsd_sparse_decode, with its scratch (status word, merge counters, split-K
// partials) in a fixed array that lives in the library itself.
//
// The array is a file-scope __device__ object of kStaticWsBytes bytes, so every
// GPU that loads this library holds that much memory until the process exits.
// Host code cannot use the array's name as an address: the first call on each
// device asks the runtime for the array's device address (cudaGetSymbolAddress)
// with that device current, checks the result and keeps it for later calls.  The kept
// address belongs to the device's primary context: after a cudaDeviceReset it is stale, and
// the entry point must not be called on that device again in the same process.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "tsd.h"
#include "tsd_args.h"
#include "tsd_plan.h"

namespace tsd {
cudaError_t launch_sparse_decode(const DecodeArgs& a, int batch, int hkv, cudaStream_t stream, bool dependent);
tsd_status prepare_sparse_decode(const tsd_kv_cache* cache, const tsd_queries* queries, const int32_t* idx,
                                 int32_t k_max, void* out, int32_t out_dtype, float* lse, DecodeArgs* a,
                                 Shapes* sh, size_t* ws_needed, size_t* zero_bytes);
}  // namespace tsd

namespace {

constexpr size_t kStaticWsBytes = 16u << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mu;
void* g_ptr[kMaxDevices] = {nullptr};

// Device address of g_static_ws on the current device (looked up once per device).
cudaError_t static_ws_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" tsd_status tsd_sparse_decode_static_ws(const tsd_kv_cache* cache, const tsd_queries* queries,
                                                  const int32_t* idx, int32_t k_max, void* out, int32_t out_dtype,
                                                  float* lse, uint32_t* status, tsd_stream_t stream) {
  using namespace tsd;
  DecodeArgs a;
  Shapes sh;
  size_t need = 0, zero = 0;
  tsd_status st = prepare_sparse_decode(cache, queries, idx, k_max, out, out_dtype, lse, &a, &sh, &need, &zero);
  if (st != TSD_OK) return st;
  if (need > kStaticWsBytes) return TSD_ERR_WORKSPACE_TOO_SMALL;
  void* base = nullptr;
  if (static_ws_address(&base) != cudaSuccess) return TSD_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: clear the status word and the merge counters
  if (cudaMemsetAsync(base, 0, zero, s) != cudaSuccess) return TSD_ERR_CUDA;
  const DecodeLayout lay = decode_layout(sh, a.nsplit);
  char* ws = static_cast<char*>(base);
  a.status = status != nullptr ? status : reinterpret_cast<uint32_t*>(ws);
  a.counters = reinterpret_cast<uint32_t*>(ws + lay.off_counters);
  a.part_ml = reinterpret_cast<float2*>(ws + lay.off_ml);
  a.part_acc = reinterpret_cast<float*>(ws + lay.off_acc);
  a.sched = reinterpret_cast<uint32_t*>(ws + 4);
  return launch_sparse_decode(a, (int)sh.batch, (int)sh.hkv, s, false) == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}
