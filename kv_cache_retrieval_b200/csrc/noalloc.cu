// hhr_decode_step_noalloc: the fused decode step for callers that cannot
// allocate device memory for a workspace.  Its scratch is a fixed-size array
// in this file, owned by the library on every device that loads it.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "hhr.h"
#include "hhr_internal.cuh"

namespace {

// Scratch shared by every call on a device; zero when the module loads.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HHR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the array's name in host code is only a host-side handle).
int32_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HHR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HHR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HHR_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HHR_OK;
}

}  // namespace

extern "C" int32_t hhr_decode_step_noalloc(const hhr_dims* dims, const void* q, const float* R,
                                           const float* W, const uint32_t* codes,
                                           const void* meta, const void* K, const void* V,
                                           int32_t n_valid, int32_t P, int32_t k, float scale,
                                           int32_t* page_idx, int32_t* tok_idx, int32_t* n_sel,
                                           float* out, void* stream) {
  const size_t need = hhr_workspace_size(dims, P, k);
  if (need == 0)  // invalid or unsupported sizes: report them as hhr_decode_step does
    return hhr_decode_step(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx,
                           tok_idx, n_sel, out, nullptr, 0, stream);
  if (need > HHR_NOALLOC_SCRATCH_BYTES) return HHR_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (int32_t st = scratch_address(&scratch)) return st;
  // every argument check first: a rejected call must not touch the scratch
  // that a call still running on the GPU may be using
  if (int32_t st = hhr::decode_step_check(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale,
                                          page_idx, tok_idx, n_sel, out, scratch,
                                          HHR_NOALLOC_SCRATCH_BYTES))
    return st;
  // The per-unit counters must start at zero (a timed-out call leaves them
  // set); the status word is left as it is until hhr_noalloc_read_status
  // reads it.  The rest of the scratch is written before it is read.
  const hhr::WsLayout L =
      hhr::ws_layout(dims->B * dims->Hkv, (dims->n_cap + dims->page - 1) / dims->page,
                     dims->Hq / dims->Hkv, hhr::hist_bins(dims->Hq / dims->Hkv, dims->bits, dims->flags));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + L.counters, 0, L.U - L.counters, s) != cudaSuccess)
    return HHR_ERR_CUDA;
  return hhr_decode_step(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx, tok_idx,
                         n_sel, out, scratch, HHR_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int32_t hhr_noalloc_read_status(void* stream) {
  void* scratch = nullptr;
  if (int32_t st = scratch_address(&scratch)) return st;
  // the status word is the scratch's first word, as in a caller workspace
  return hhr_read_status(scratch, stream);
}
