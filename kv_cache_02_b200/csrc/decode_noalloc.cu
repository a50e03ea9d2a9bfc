// gqa_decode_noalloc: gqa_decode with the split-KV partials kept in a static
// device array of this library instead of a caller-owned workspace, for
// callers that cannot allocate device memory at decode time (include/gqa.h
// lists who and why). It adds no kernel: it hands the array's device address
// to gqa_decode as the workspace.
#include <cuda.h>
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
unsigned long long g_scratch_ctx[kMaxDevices] = {0};  // the context the address belongs to
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The process-unique id of this thread's current CUDA context, or 0 when
// there is none (or the driver cannot tell). A device reset destroys the
// context, and with it the array's address; the next context has a new id.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Set-up, with the device current: look up the device address of the
// scratch. Done once per device; again only if the device's context is not
// the one the address was found in (a reset), or cannot be told.
int scratch_on_current_device(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the lookup made the device's context current
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
