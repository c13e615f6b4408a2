// kvq_decode_attention_noalloc: decode + combine with library-owned scratch.
//
// Some callers cannot call cudaMalloc at decode time: code running inside a
// memory pool or arena that hands out every byte it owns up front, callers
// that must not touch the allocator while a CUDA graph is being captured
// elsewhere in the process, and host languages or runtimes that only pass
// pointers they were given.  For them this entry point needs no workspace:
// the split partials go to a fixed-size array in device memory that this
// file declares at file scope.
//
// The array (kStaticScratchBytes) is reserved in a GPU's memory when the CUDA
// runtime loads this library's module on that GPU -- at context creation under
// eager module loading (CUDA_MODULE_LOADING=EAGER), at the first use of the
// module under lazy loading -- and stays until the process exits.  All calls on
// one GPU share it and it keeps the previous call's contents; every entry the
// decode kernel reads back is written first in the same call, so nothing needs
// clearing.  Two calls whose kernels overlap on the GPU (different streams,
// no ordering between them) race on the array and give wrong results.
//
// In host code the array's name is only a host-side stand-in, not a device
// address; the device address is looked up with cudaGetSymbolAddress once per
// GPU, with that GPU current, on the first call made there.  That first call
// should therefore come before any stream capture.  The address is kept for the
// life of the process: after cudaDeviceReset (or anything else that destroys
// the device's primary context) it is stale, and this entry point must not be
// used again in that process.
#include <mutex>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per GPU
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_dev_ptr[kMaxDevices] = {};

kvq_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return KVQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_dev_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_last_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return KVQ_ERR_CUDA;
    }
    g_scratch_dev_ptr[dev] = p;
  }
  *out = g_scratch_dev_ptr[dev];
  return KVQ_OK;
}

}  // namespace
}  // namespace kvq

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* k_cache,
                                                   const void* v_cache, const void* q, int32_t batch,
                                                   int64_t ctx_len, float softmax_scale, int32_t n_splits,
                                                   float* out, void* cuda_stream) {
  kvq_status st = kvq_check_desc(desc);
  if (st != KVQ_OK) return st;
  if (!out || (reinterpret_cast<uintptr_t>(out) % 16) != 0) return KVQ_ERR_INVALID;
  if (n_splits < 0 || n_splits > kvq::kMaxSplits) return KVQ_ERR_INVALID;
  int32_t S = n_splits;
  if (S == 0) {
    // automatic count, lowered to the largest count whose partials fit the scratch
    S = kvq_auto_splits(desc, batch, ctx_len);
    if (S == 0) return KVQ_ERR_INVALID;
    while (S > 1 && kvq_workspace_bytes(desc, batch, S) > kvq::kStaticScratchBytes) --S;
  }
  const size_t need = kvq_workspace_bytes(desc, batch, S);
  if (need == 0) return KVQ_ERR_INVALID;
  if (need > kvq::kStaticScratchBytes) return KVQ_ERR_WORKSPACE;
  void* ws = nullptr;
  st = kvq::scratch_on_current_device(&ws);
  if (st != KVQ_OK) return st;
  st = kvq_decode_attention(desc, k_cache, v_cache, q, batch, ctx_len, softmax_scale, S, ws,
                            kvq::kStaticScratchBytes, cuda_stream);
  if (st != KVQ_OK) return st;
  return kvq_combine(desc, ws, kvq::kStaticScratchBytes, batch, ctx_len, S, out, cuda_stream);
}
