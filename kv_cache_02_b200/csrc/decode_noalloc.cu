// gqa_decode_noalloc: gqa_decode with the split-KV partials kept in a static
// device array of this library instead of a caller-owned workspace, for
// callers that cannot allocate device memory at decode time (include/gqa.h
// lists who and why). It adds no kernel: it hands the array's device address
// to gqa_decode as the workspace.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "../../include/gqa.h"

// The scratch. Every GPU that loads the library holds GQA_NOALLOC_SCRATCH_BYTES
// of it until the process exits. In host code this name is only a host-side
// stand-in: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GQA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Set-up, once per device and with that device current: look up the device
// address of the scratch.
int scratch_on_current_device(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return GQA_OK;
}

}  // namespace

extern "C" int gqa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* seqlens, int B, int H, int K, int S_max, int d, float scale,
                                  int num_splits, gqa_dtype dtype, gqa_stream_t stream) {
  const size_t need = gqa_decode_workspace_bytes(B, H, K, S_max, d, num_splits);
  if (need > (size_t)GQA_NOALLOC_SCRATCH_BYTES) return GQA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (need > 0) {
    const int rc = scratch_on_current_device(&scratch);
    if (rc != GQA_OK) return rc;
    scratch_bytes = GQA_NOALLOC_SCRATCH_BYTES;
  }
  return gqa_decode(out, q, k_cache, v_cache, seqlens, B, H, K, S_max, d, scale, num_splits, scratch, scratch_bytes,
                    dtype, stream);
}
