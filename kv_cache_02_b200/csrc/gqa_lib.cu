// libgqa.so: the C ABI declared in include/gqa.h.
//
// Host side only validates arguments, plans the launch and encodes TMA
// descriptors; every step of the computation runs in the kernels included
// below. The library allocates no device memory: callers own all buffers,
// including the decode workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <random>

#include "../../include/gqa.h"
#include "append_meanpool.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "decode_wide.cuh"
#include "prefill.cuh"
#include "prefill_pair.cuh"
#include "kv_proj.cuh"

namespace {

using gqa::DecodeParams;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A runtime query that may fail (no GPU in the process) leaves its error as
// the thread's last CUDA error. It is cleared only if no error was pending
// before the query, so a caller's own pending error is never swallowed.
struct QueryErrorScope {
  const cudaError_t before = cudaPeekAtLastError();
  void clear_own() const {
    if (before == cudaSuccess) cudaGetLastError();
  }
};

int current_device() {
  int dev = 0;
  const QueryErrorScope scope;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    scope.clear_own();
    return -1;
  }
  return dev;
}

// Per-device values computed once. Host threads may plan launches at the
// same time: the entries are atomics (0 = not yet known), and two threads
// that both compute one store the same value.
using DeviceCache = std::atomic<int>[kMaxDevices];

int sm_count(int dev) {
  static DeviceCache cache{};
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_acquire);
  if (n == 0) {
    const QueryErrorScope scope;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      scope.clear_own();
      n = 148;
    }
    cache[dev].store(n, std::memory_order_release);
  }
  return n;
}

// cuTensorMapEncodeTiled from the driver, found through the runtime so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over rows of `cols` elements, box = box_rows x 64 columns
// (128 bytes), 128-byte swizzle. Rows past `rows` read as zero.
bool encode_rows_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, 128] int8 codes, 128-byte rows (one swizzle span), box of box_rows rows.
bool encode_rows_u8(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [units, S_max] float scales (row stride S_max * 4 bytes, a multiple of 16), box of 64 scales of one unit.
bool encode_scales(CUtensorMap* map, const float* base, uint64_t units, uint64_t S_max) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {S_max, units};
  cuuint64_t strides[1] = {S_max * 4};
  cuuint32_t box[2] = {(cuuint32_t)gqa::kDecTileKeys, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// ----------------------------------------------------------------------------
// decode launch plan

struct DecodePlan {
  bool wide = false;   // bf16, d 128, G a multiple of 64: the tcgen05 decode (64 heads per CTA)
  int chunk = 0;       // keys per split (multiple of the tile)
  int nsplit = 1;      // splits per (b, g)
  int hslices = 1;     // head slices per (b, g)
  long long grid = 0;  // bf16: persistent CTAs; f32: one CTA per work item
  size_t ws_bytes = 0;
  size_t ws_ml_off = 0, ws_queue_off = 0;
};

// A 40-bit tag that differs on every decode call of this process and, being
// seeded at random, from the tags of other processes: a work counter left by
// an earlier call (or uninitialised memory) does not match it.
unsigned long long next_call_tag() {
  static std::atomic<unsigned long long> counter{0};
  static unsigned long long seed = [] {
    std::random_device rd;
    const unsigned long long t =
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
    return ((((unsigned long long)rd()) << 32) ^ rd() ^ (t * 0x9E3779B97F4A7C15ull)) | 1ull;
  }();
  const unsigned long long t = (seed + 2ull * counter.fetch_add(1)) & ((1ull << 40) - 1);
  return t ? t : 1ull;
}

bool valid_decode_shape(int B, int H, int K, int S_max, int d, bool paged = false) {
  if (B < 0 || H <= 0 || K <= 0 || S_max <= 0) return false;
  if (H % K != 0) return false;
  if (d != 64 && d != 128) return false;
  if (!paged && (long long)B * K * S_max >= (1ll << 31)) return false;  // TMA row coordinate is int32
  if ((long long)B * H >= (1ll << 31)) return false;
  return true;
}

// A paged cache: a pool of num_blocks blocks [K, block_size, d] and a block
// table [B, max_blocks] (see DecodeParams).
struct PagedCache {
  const int32_t* table = nullptr;
  int num_blocks = 0, block_size = 0, max_blocks = 0;
};

bool valid_paged(const PagedCache& pc, int B, int K) {
  if (pc.num_blocks <= 0 || pc.block_size <= 0 || pc.max_blocks <= 0) return false;
  if (pc.block_size % 16 != 0) return false;  // a 16-row TMA box never straddles blocks
  if ((long long)pc.max_blocks * pc.block_size >= (1ll << 31)) return false;
  if ((long long)pc.num_blocks * K * pc.block_size >= (1ll << 31)) return false;  // TMA row coordinate
  if ((long long)B * pc.max_blocks >= (1ll << 31)) return false;
  return true;
}

// Resident persistent decode CTAs per SM for head dim D (2 on B200), cached per device.
template <int D>
int decode_ctas_per_sm(int dev) {
  static DeviceCache cache{};
  if (dev < 0 || dev >= kMaxDevices) return 2;
  int n = cache[dev].load(std::memory_order_acquire);
  if (n == 0) {
    using C = gqa::DecCfg<D>;
    const QueryErrorScope scope;
    if (cudaFuncSetAttribute(gqa::decode_bf16_kernel<D, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gqa::decode_bf16_kernel<D, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gqa::decode_bf16_kernel<D, false, false>, gqa::kDecThreads,
                                                      C::kSmemBytes) != cudaSuccess ||
        n <= 0) {
      scope.clear_own();  // no GPU here: plan with the B200 figure
      n = 2;
    }
    cache[dev].store(n, std::memory_order_release);
  }
  return n;
}

// Resident 8-bit-cache decode CTAs per SM (2 on B200), cached per device.
int decode_i8_ctas_per_sm(int dev) {
  static DeviceCache cache{};
  if (dev < 0 || dev >= kMaxDevices) return 2;
  int n = cache[dev].load(std::memory_order_acquire);
  if (n == 0) {
    using C = gqa::DecCfg<128, true>;
    const QueryErrorScope scope;
    if (cudaFuncSetAttribute(gqa::decode_bf16_kernel<128, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gqa::decode_bf16_kernel<128, false, true>,
                                                      gqa::kDecThreads, C::kSmemBytes) != cudaSuccess ||
        n <= 0) {
      scope.clear_own();
      n = 2;
    }
    cache[dev].store(n, std::memory_order_release);
  }
  return n;
}

// Resident wide-group decode CTAs per SM (1 on B200), cached per device.
int wide_ctas_per_sm(int dev) {
  static DeviceCache cache{};
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int n = cache[dev].load(std::memory_order_acquire);
  if (n == 0) {
    const QueryErrorScope scope;
    if (cudaFuncSetAttribute(gqa::decode_wide_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gqa::WideCfg::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gqa::decode_wide_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gqa::WideCfg::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gqa::decode_wide_kernel<false>, gqa::kWideThreads,
                                                      gqa::WideCfg::kSmemBytes) != cudaSuccess ||
        n <= 0) {
      scope.clear_own();
      n = 1;
    }
    cache[dev].store(n, std::memory_order_release);
  }
  return n;
}

// int8: the 8-bit cache (narrow-group kernel only).
DecodePlan plan_decode(int B, int H, int K, int S_max, int d, int num_splits, gqa_dtype dt, int sms,
                       bool int8 = false, bool paged = false) {
  DecodePlan pl;
  const int G = H / K;
  pl.wide = !int8 && dt == GQA_BF16 && d == 128 && G % gqa::kWideHeads == 0;
  const int heads_per_cta =
      pl.wide ? gqa::kWideHeads : (dt == GQA_BF16 ? gqa::kDecHeadsPerCta : gqa::kDecF32HeadsPerCta);
  const int tile = pl.wide ? gqa::kWideKeys : 64;
  pl.hslices = (G + heads_per_cta - 1) / heads_per_cta;
  const long long units = (long long)B * K * pl.hslices;
  const int max_splits = std::min((S_max + tile - 1) / tile, gqa::kMaxCombineSplits);
  int splits;
  if (num_splits > 0) {
    splits = std::min(num_splits, max_splits);
  } else {
    // narrow groups: about eight small work items per SM (their partials are
    // small), twelve for bf16 batches of many units, where the finer items
    // shorten the tail (split sweeps: the 70B ragged batch 2 % faster, the
    // Llama-3-8B layer within 1 %), six for the 8-bit cache, whose consumers
    // pay more per item (split sweeps: the Llama-3-8B shape 0.72 -> 0.74 of
    // the copy bandwidth at 14 splits instead of 19, the 70B ragged batch
    // 0.84 -> 0.87 at 4 instead of 5); wide groups: about one item per SM,
    // since a 64-head partial is 32 KB; never below 256 keys per split, nor
    // below 448 for a paged cache, whose producer loads an item's window of
    // the block table at its start (Llama-3-8B layer at block size 16: 0.86
    // of the copy bandwidth with 320-key splits, 0.89 with 448)
    const long long per_sm = int8 ? 6 : (units >= 32 ? 12 : 8);
    const long long target = pl.wide ? (long long)sms : per_sm * sms;
    const int min_chunk = paged ? 448 : 256;
    splits = (int)std::max<long long>(1, (target + units - 1) / std::max<long long>(units, 1));
    splits = std::min(splits, std::max(1, (S_max + min_chunk - 1) / min_chunk));
    splits = std::min(splits, max_splits);
  }
  int chunk = (S_max + splits - 1) / splits;
  chunk = (chunk + tile - 1) / tile * tile;
  pl.chunk = chunk;
  pl.nsplit = (S_max + chunk - 1) / chunk;
  const size_t parts = (size_t)B * K * pl.nsplit * G;
  const size_t part_bytes = pl.nsplit > 1 ? parts * d * sizeof(float) + parts * sizeof(float2) : 0;
  pl.ws_ml_off = parts * d * sizeof(float);
  if (dt == GQA_BF16) {
    // persistent CTAs that take work items from a counter in the workspace
    const int dev = current_device();
    const int per_sm = pl.wide ? wide_ctas_per_sm(dev)
                               : int8 ? decode_i8_ctas_per_sm(dev)
                                      : (d == 128 ? decode_ctas_per_sm<128>(dev) : decode_ctas_per_sm<64>(dev));
    const long long items = units * pl.nsplit;
    pl.grid = std::max<long long>(1, std::min<long long>(items, (long long)per_sm * sms));
    if (items + pl.grid >= (1ll << 24)) {  // beyond the work counter
      pl.ws_bytes = (size_t)-1;
      return pl;
    }
    pl.ws_queue_off = (part_bytes + 15) / 16 * 16;
    pl.ws_bytes = pl.ws_queue_off + 16;
    return pl;
  }
  pl.grid = units * pl.nsplit;
  pl.ws_bytes = part_bytes;
  return pl;
}

// rows: of the [rows, D] view of the cache (B * K * S_max) or the pool (num_blocks * K * block_size)
template <int D>
int launch_decode_bf16(const DecodePlan& pl, const DecodeParams& p, const void* kc, const void* vc, uint64_t rows,
                       cudaStream_t st) {
  CUtensorMap tk64, tv64, tk, tv;  // 64-row boxes for full tiles, 16-row boxes for the rest
  if (!encode_rows_bf16(&tk64, kc, rows, D, gqa::kDecTileKeys) ||
      !encode_rows_bf16(&tv64, vc, rows, D, gqa::kDecTileKeys) ||
      !encode_rows_bf16(&tk, kc, rows, D, gqa::kDecBoxRows) || !encode_rows_bf16(&tv, vc, rows, D, gqa::kDecBoxRows))
    return GQA_ERR_CUDA;
  using C = gqa::DecCfg<D>;
  decode_ctas_per_sm<D>(current_device());  // sets the shared-memory attribute once per device
  // (the scale maps of the 8-bit kernel are unused here: the K maps stand in)
  // a programmatic dependent launch: see decode_bf16_kernel on what it does before the grid dependency
  if (p.block_table)
    return gqa::launch_kernel(gqa::decode_bf16_kernel<D, true, false>, (unsigned)pl.grid, gqa::kDecThreads,
                              C::kSmemBytes, st, true, tk64, tv64, tk, tv, tk64, tv64, p);
  return gqa::launch_kernel(gqa::decode_bf16_kernel<D, false, false>, (unsigned)pl.grid, gqa::kDecThreads,
                            C::kSmemBytes, st, true, tk64, tv64, tk, tv, tk64, tv64, p);
}

// The 8-bit cache: codes [units * S_max, 128] int8, scales [units, S_max] float.
int launch_decode_i8(const DecodePlan& pl, const DecodeParams& p, const void* kc, const void* vc, const float* ks,
                     const float* vs, uint64_t units, uint64_t S_max, cudaStream_t st) {
  CUtensorMap tk64, tv64, tk, tv, tks, tvs;
  const uint64_t rows = units * S_max;
  if (!encode_rows_u8(&tk64, kc, rows, gqa::kDecTileKeys) || !encode_rows_u8(&tv64, vc, rows, gqa::kDecTileKeys) ||
      !encode_rows_u8(&tk, kc, rows, gqa::kDecBoxRows) || !encode_rows_u8(&tv, vc, rows, gqa::kDecBoxRows) ||
      !encode_scales(&tks, ks, units, S_max) || !encode_scales(&tvs, vs, units, S_max))
    return GQA_ERR_CUDA;
  using C = gqa::DecCfg<128, true>;
  decode_i8_ctas_per_sm(current_device());  // sets the shared-memory attribute once per device
  return gqa::launch_kernel(gqa::decode_bf16_kernel<128, false, true>, (unsigned)pl.grid, gqa::kDecThreads,
                            C::kSmemBytes, st, true, tk64, tv64, tk, tv, tks, tvs, p);
}

int launch_decode_wide(const DecodePlan& pl, const DecodeParams& p, const void* q, const void* kc, const void* vc,
                       int B, int H, uint64_t rows, cudaStream_t st) {
  CUtensorMap tq, tk64, tv64, tk16, tv16;
  if (!encode_rows_bf16(&tq, q, (uint64_t)B * H, 128, gqa::kWideHeads) ||
      !encode_rows_bf16(&tk64, kc, rows, 128, gqa::kWideBox) || !encode_rows_bf16(&tv64, vc, rows, 128, gqa::kWideBox) ||
      !encode_rows_bf16(&tk16, kc, rows, 128, gqa::kDecBoxRows) ||
      !encode_rows_bf16(&tv16, vc, rows, 128, gqa::kDecBoxRows))
    return GQA_ERR_CUDA;
  wide_ctas_per_sm(current_device());  // sets the shared-memory attribute once per device
  if (p.block_table)
    return gqa::launch_kernel(gqa::decode_wide_kernel<true>, (unsigned)pl.grid, gqa::kWideThreads,
                              gqa::WideCfg::kSmemBytes, st, true, tq, tk64, tv64, tk16, tv16, p);
  return gqa::launch_kernel(gqa::decode_wide_kernel<false>, (unsigned)pl.grid, gqa::kWideThreads,
                            gqa::WideCfg::kSmemBytes, st, true, tq, tk64, tv64, tk16, tv16, p);
}

template <int D>
int launch_decode_f32(const DecodePlan& pl, const DecodeParams& p, const void* kc, const void* vc,
                      cudaStream_t st) {
  return gqa::launch_kernel(gqa::decode_f32_kernel<D>, (unsigned)pl.grid, gqa::kDecF32Threads, 0, st, false,
                            static_cast<const float*>(kc), static_cast<const float*>(vc), p);
}

int launch_prefill(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache, int B, int S,
                   int H, int K, int S_max, int d, float scale, cudaStream_t st, int sms);

int grid_for(long long work_items, int threads, int sms) {
  long long blocks = (work_items + threads - 1) / threads;
  long long cap = (long long)sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

int launch_prefill(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache, int B, int S,
                   int H, int K, int S_max, int d, float scale, cudaStream_t st, int sms) {
  auto fn = reinterpret_cast<gqa::PfEncodeFn>(encode_fn());
  if (!fn) return GQA_ERR_CUDA;
  if ((long long)B * S >= (1ll << 31)) return GQA_ERR_SHAPE;
  if (k_cache && (long long)B * K * S_max >= (1ll << 31)) return GQA_ERR_SHAPE;  // TMA row coordinate
  if ((H / K) % 2 == 0)  // two heads of a group per work unit; the cache write is fused
    return d == 128 ? gqa::launch_prefill_pair_d<128>(fn, out, q, k, v, k_cache, v_cache, B, S, H, K, S_max, scale,
                                                      st, sms)
                    : gqa::launch_prefill_pair_d<64>(fn, out, q, k, v, k_cache, v_cache, B, S, H, K, S_max, scale, st,
                                                     sms);
  int rc = d == 128 ? gqa::launch_prefill_d<128>(fn, out, q, k, v, B, S, H, K, scale, st)
                    : gqa::launch_prefill_d<64>(fn, out, q, k, v, B, S, H, K, scale, st);
  if (rc != GQA_OK || !k_cache) return rc;
  const int cpr = d * 2 / 16;
  const long long work = 2ll * B * S * K * cpr;
  return gqa::launch_kernel(gqa::kv_write_prompt_kernel, (unsigned)grid_for(work, 256, sms), 256, 0, st, false,
                            static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<const uint4*>(k),
                            static_cast<const uint4*>(v), B, S, K, S_max, cpr);
}

// Varlen: packed [T, heads, d] tokens of B sequences given by cu_seqlens.
int launch_prefill_varlen(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache,
                          const int32_t* cu_seqlens, int B, int T, int H, int K, int S_max, int d, float scale,
                          cudaStream_t st, int sms) {
  auto fn = reinterpret_cast<gqa::PfEncodeFn>(encode_fn());
  if (!fn) return GQA_ERR_CUDA;
  if (k_cache && (long long)B * K * S_max >= (1ll << 31)) return GQA_ERR_SHAPE;  // TMA row coordinate
  if ((H / K) % 2 == 0)
    return d == 128 ? gqa::launch_prefill_pair_d<128>(fn, out, q, k, v, k_cache, v_cache, B, 0, H, K, S_max, scale,
                                                      st, sms, cu_seqlens, T)
                    : gqa::launch_prefill_pair_d<64>(fn, out, q, k, v, k_cache, v_cache, B, 0, H, K, S_max, scale, st,
                                                     sms, cu_seqlens, T);
  int rc = d == 128 ? gqa::launch_prefill_d<128>(fn, out, q, k, v, B, 0, H, K, scale, st, cu_seqlens, T)
                    : gqa::launch_prefill_d<64>(fn, out, q, k, v, B, 0, H, K, scale, st, cu_seqlens, T);
  if (rc != GQA_OK || !k_cache) return rc;
  const int cpr = d * 2 / 16;
  const long long work = 2ll * T * K * cpr;
  return gqa::launch_kernel(gqa::kv_write_prompt_varlen_kernel, (unsigned)grid_for(work, 256, sms), 256, 0, st,
                            false, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                            static_cast<const uint4*>(k), static_cast<const uint4*>(v), cu_seqlens, B, T, K, S_max,
                            cpr);
}

// Fused K/V projection: d_model is split over CTAs (powers of two, at least
// 4 pipeline steps each) while the token tiles x heads leave SMs idle.
struct ProjPlan {
  bool small = false;
  int splits = 1;
  long long grid = 0;
  size_t ws_bytes = 0;
};

// small: at most 16 tokens (a decode step), the weight-streaming GEMV: one
// CTA per 16 W_KV rows over all of d_model, no split, no workspace.
// Otherwise the token-tile GEMM, d_model split while tiles leave SMs idle.
ProjPlan plan_proj(long long M, int K, int d, int d_model, int sms) {
  ProjPlan pl;
  pl.small = M <= gqa::kPsTok;
  if (pl.small) {
    pl.grid = (long long)K * 2 * d / gqa::kGvRows;
    return pl;
  }
  const int ksteps = d_model / gqa::kPjBK;
  const long long base = (M + gqa::kPjBM - 1) / gqa::kPjBM * K;
  while (base * pl.splits < sms && ksteps % (pl.splits * 2) == 0 && ksteps / (pl.splits * 2) >= 4 &&
         pl.splits * 2 <= gqa::kPjMaxSplits)
    pl.splits *= 2;
  pl.grid = base * pl.splits;
  pl.ws_bytes = pl.splits > 1 ? (size_t)pl.splits * (size_t)M * K * 2 * d * sizeof(float) : 0;
  return pl;
}

// A 3-D bf16 view of a row-major [rows, cols] matrix as (64 columns, rows,
// cols / 64 blocks of 64 columns), box (64, box_rows, box_blocks), 128-byte
// swizzle: one load brings box_rows rows x 64 box_blocks columns, block-major.
bool encode_row_blocks_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                            uint32_t box_blocks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NT>
int launch_proj_gemv(const ProjPlan& pl, const gqa::ProjParams& p, const void* x, const void* w, int d_model,
                     cudaStream_t st) {
  using G = gqa::GvCfg<NT>;
  CUtensorMap tx, tw;
  if (!encode_row_blocks_bf16(&tx, x, (uint64_t)p.M, (uint64_t)d_model, 8 * NT, gqa::kGvCols / 64) ||
      !encode_row_blocks_bf16(&tw, w, (uint64_t)p.K * 2 * D, (uint64_t)d_model, gqa::kGvRows, gqa::kGvCols / 64))
    return GQA_ERR_CUDA;
  static DeviceCache configured{};
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && configured[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(gqa::kv_proj_gemv_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::kSmemBytes) != cudaSuccess)
      return GQA_ERR_CUDA;
    configured[dev].store(1, std::memory_order_release);
  }
  // a programmatic dependent launch: it warms L2 with its W_KV rows before the grid dependency
  return gqa::launch_kernel(gqa::kv_proj_gemv_kernel<D, NT>, (unsigned)pl.grid, G::kThreads, G::kSmemBytes, st, true,
                            tx, tw, p, d_model);
}

bool valid_proj(int B, int T, int K, int S_max, int d, int d_model) {
  if (B < 0 || T <= 0 || K <= 0 || S_max <= 0 || d_model <= 0) return false;
  if ((d != 64 && d != 128) || d_model % gqa::kPjBK != 0) return false;
  if ((long long)B * T >= (1ll << 31) || (long long)K * 2 * d >= (1ll << 31)) return false;
  return true;
}

template <int D>
int launch_proj_d(const ProjPlan& pl, gqa::ProjParams p, const void* x, const void* w, int d_model, cudaStream_t st,
                  int sms) {
  using C = gqa::PjCfg<D>;
  if (pl.small)
    return p.M <= 8 ? launch_proj_gemv<D, 1>(pl, p, x, w, d_model, st) : launch_proj_gemv<D, 2>(pl, p, x, w, d_model, st);
  CUtensorMap tx, tw;
  if (!encode_rows_bf16(&tx, x, (uint64_t)p.M, (uint64_t)d_model, gqa::kPjBM) ||
      !encode_rows_bf16(&tw, w, (uint64_t)p.K * C::kN, (uint64_t)d_model, C::kN))
    return GQA_ERR_CUDA;
  static DeviceCache configured{};
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && configured[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(gqa::kv_proj_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return GQA_ERR_CUDA;
    configured[dev].store(1, std::memory_order_release);
  }
  {
    const int rc =
        gqa::launch_kernel(gqa::kv_proj_kernel<D>, (unsigned)pl.grid, gqa::kPjThreads, C::kSmemBytes, st, false, tx, tw, p);
    if (rc != GQA_OK) return rc;
  }
  if (pl.splits > 1) {  // as a programmatic dependent launch: its launch overlaps the GEMM
    const long long work = (long long)p.M * p.K * C::kN;
    return gqa::launch_kernel(gqa::kv_proj_finalize_kernel<D>, (unsigned)grid_for(work, 256, sms), 256, 0, st, true,
                              p);
  }
  return GQA_OK;
}

}  // namespace

// ============================================================================
// C ABI

extern "C" {

const char* gqa_status_string(int status) {
  switch (status) {
    case GQA_OK: return "GQA_OK";
    case GQA_ERR_INVALID_ARG: return "GQA_ERR_INVALID_ARG";
    case GQA_ERR_SHAPE: return "GQA_ERR_SHAPE";
    case GQA_ERR_ALIGN: return "GQA_ERR_ALIGN";
    case GQA_ERR_CUDA: return "GQA_ERR_CUDA";
    case GQA_ERR_DEVICE: return "GQA_ERR_DEVICE";
    case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED";
    case GQA_ERR_SCRATCH_LIMIT: return "GQA_ERR_SCRATCH_LIMIT";
    default: return "GQA_ERR_UNKNOWN";
  }
}

size_t gqa_decode_workspace_bytes(int B, int H, int K, int S_max, int d, int num_splits) {
  if (!valid_decode_shape(B, H, K, S_max, d) || num_splits < 0) return 0;
  const int dev = current_device();
  // the plan does not depend on the dtype except through the head slicing,
  // which does not change the workspace size; take the larger of the two
  const DecodePlan a = plan_decode(B, H, K, S_max, d, num_splits, GQA_BF16, sm_count(dev));
  const DecodePlan b = plan_decode(B, H, K, S_max, d, num_splits, GQA_F32, sm_count(dev));
  if (a.ws_bytes == (size_t)-1) return 0;
  return std::max(a.ws_bytes, b.ws_bytes);
}

}  // extern "C"

namespace {

template <typename OutT, int D, int NT, int CS>
int launch_combine_t(void* out, const DecodeParams& p, const int32_t* seqlens, int H, int K, int S_max, int G,
                     int chunk, int nsplit, int skip_single, long long units, cudaStream_t st) {
  return gqa::launch_kernel(gqa::decode_combine_kernel<OutT, D, NT, CS>, (unsigned)(units * CS), NT, 0, st, true,
                            static_cast<OutT*>(out), (const float*)p.ws_o, (const float2*)p.ws_ml, seqlens, p.len_add,
                            H, K, S_max, G, chunk, nsplit, skip_single);
}

// Few splits: one CTA of 128 threads per (b, h). Many splits: four CTAs of
// 256 threads per (b, h), a quarter of the columns each, so that more SMs
// share the partial rows and all of them are loaded in one round.
template <typename OutT, int D>
int launch_combine_d(void* out, const DecodeParams& p, const int32_t* seqlens, int H, int K, int S_max, int G,
                             int chunk, int nsplit, int skip_single, bool many, long long units, cudaStream_t st) {
  return many ? launch_combine_t<OutT, D, 256, 4>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single, units,
                                                  st)
              : launch_combine_t<OutT, D, 128, 1>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single, units,
                                                  st);
}

int launch_combine(void* out, const DecodeParams& p, const int32_t* seqlens, int H, int K, int S_max, int G,
                           int chunk, int nsplit, int skip_single, int d, gqa_dtype dt, bool many, long long units,
                           cudaStream_t st) {
  if (dt == GQA_BF16)
    return d == 128 ? launch_combine_d<__nv_bfloat16, 128>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single,
                                                           many, units, st)
                    : launch_combine_d<__nv_bfloat16, 64>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single,
                                                          many, units, st);
  return d == 128 ? launch_combine_d<float, 128>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single, many,
                                                 units, st)
                  : launch_combine_d<float, 64>(out, p, seqlens, H, K, S_max, G, chunk, nsplit, skip_single, many,
                                                units, st);
}

// gqa_kv_append, and with a paged cache gqa_kv_append_paged (S_max = max_blocks * block_size).
int kv_append_impl(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos, int B,
                   int K, int S_max, int d, gqa_dtype dtype, gqa_stream_t stream, const PagedCache* pc) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (B < 0 || K <= 0 || S_max <= 0) return GQA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return GQA_ERR_SHAPE;
  if (B == 0) return GQA_OK;
  if (!k_cache || !v_cache || !k_new || !v_new || !pos) return GQA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new)) return GQA_ERR_ALIGN;
  const int elt = dtype == GQA_F32 ? 4 : 2;
  const int cpr = d * elt / 16;
  const long long work = 2ll * B * K * cpr;
  const int dev = current_device();
  const int grid = grid_for(work, 256, sm_count(dev));
  return gqa::launch_kernel(gqa::kv_append_kernel, (unsigned)grid, 256, 0, (cudaStream_t)stream, false,
                            static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                            static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), pos, B, K, S_max, cpr,
                            pc ? pc->table : nullptr, pc ? pc->max_blocks : 0, pc ? pc->block_size : 0,
                            pc ? pc->num_blocks : 0);
}

// gqa_decode, and with append != 0 gqa_decode_append (seqlens then holds pos);
// with a paged cache (pc != null) their paged forms, S_max = max_blocks * block_size.
int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, int B,
                int H, int K, int S_max, int d, float scale, int num_splits, void* workspace, size_t workspace_bytes,
                gqa_dtype dtype, gqa_stream_t stream, const void* k_new, const void* v_new, int append,
                const PagedCache* pc = nullptr, const float* k_scales = nullptr, const float* v_scales = nullptr) {
  const bool int8 = k_scales != nullptr || v_scales != nullptr;  // caches of 8-bit codes with per-row scales
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (num_splits < 0 || B < 0 || H <= 0 || K <= 0 || S_max <= 0) return GQA_ERR_INVALID_ARG;
  if (!valid_decode_shape(B, H, K, S_max, d, pc != nullptr)) return GQA_ERR_SHAPE;
  if (pc && !valid_paged(*pc, B, K)) return GQA_ERR_SHAPE;
  if (pc && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;  // the paged forms stream bf16 by TMA
  if (int8 && (d != 128 || dtype != GQA_BF16 || pc || append)) return GQA_ERR_UNSUPPORTED;
  if (int8 && S_max % 4 != 0) return GQA_ERR_SHAPE;  // a scale row must start on 16 bytes
  if (B == 0) return GQA_OK;
  if (!out || !q || !k_cache || !v_cache || !seqlens || (pc && !pc->table)) return GQA_ERR_INVALID_ARG;
  if (int8 && (!k_scales || !v_scales)) return GQA_ERR_INVALID_ARG;
  if (int8 && (!aligned16(k_scales) || !aligned16(v_scales))) return GQA_ERR_ALIGN;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return GQA_ERR_ALIGN;
  if (append && (!k_new || !v_new)) return GQA_ERR_INVALID_ARG;
  if (append && (!aligned16(k_new) || !aligned16(v_new))) return GQA_ERR_ALIGN;
  const int dev = current_device();
  const DecodePlan pl = plan_decode(B, H, K, S_max, d, num_splits, dtype, sm_count(dev), int8, pc != nullptr);
  if (pl.ws_bytes == (size_t)-1) return GQA_ERR_SHAPE;  // more work items than the work counter holds
  if (pl.ws_bytes > 0) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return GQA_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return GQA_ERR_ALIGN;
  }
  const int G = H / K;
  cudaStream_t st = (cudaStream_t)stream;
  if (append && (dtype != GQA_BF16 || pl.wide)) {  // the append as its own launch, then the decode
    const int rc = kv_append_impl(const_cast<void*>(k_cache), const_cast<void*>(v_cache), k_new, v_new, seqlens, B,
                                  K, S_max, d, dtype, stream, pc);
    if (rc != GQA_OK) return rc;
  }
  DecodeParams p;
  const bool fused_append = append && dtype == GQA_BF16 && !pl.wide;
  p.k_new = fused_append ? k_new : nullptr;
  p.v_new = fused_append ? v_new : nullptr;
  p.k_cache_w = const_cast<void*>(k_cache);
  p.v_cache_w = const_cast<void*>(v_cache);
  p.len_add = append ? 1 : 0;
  p.q = q;
  p.out = out;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + pl.ws_ml_off);
  p.ws_queue = dtype == GQA_BF16 ? reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) +
                                                                         pl.ws_queue_off)
                                 : nullptr;
  p.nitems = (int)((long long)B * K * pl.hslices * pl.nsplit);
  p.tag = next_call_tag();
  p.seqlens = seqlens;
  p.B = B;
  p.H = H;
  p.K = K;
  p.S_max = S_max;
  p.G = G;
  p.hslices = pl.hslices;
  p.chunk = pl.chunk;
  p.nsplit = pl.nsplit;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = pc ? pc->table : nullptr;
  p.max_blocks = pc ? pc->max_blocks : 0;
  p.block_size = pc ? pc->block_size : 0;
  p.num_blocks = pc ? pc->num_blocks : 0;
  const uint64_t rows = pc ? (uint64_t)pc->num_blocks * K * pc->block_size : (uint64_t)B * K * S_max;
  int rc;
  if (int8)
    rc = launch_decode_i8(pl, p, k_cache, v_cache, k_scales, v_scales, (uint64_t)B * K, (uint64_t)S_max, st);
  else if (pl.wide)
    rc = launch_decode_wide(pl, p, q, k_cache, v_cache, B, H, rows, st);
  else if (dtype == GQA_BF16)
    rc = d == 128 ? launch_decode_bf16<128>(pl, p, k_cache, v_cache, rows, st)
                  : launch_decode_bf16<64>(pl, p, k_cache, v_cache, rows, st);
  else
    rc = d == 128 ? launch_decode_f32<128>(pl, p, k_cache, v_cache, st)
                  : launch_decode_f32<64>(pl, p, k_cache, v_cache, st);
  if (rc != GQA_OK || pl.nsplit == 1) return rc;
  // the split-KV combine, as a programmatic dependent launch: its launch
  // overlaps the decode kernel, and it waits for that grid before reading
  const int skip_single = dtype == GQA_BF16 ? 1 : 0;  // bf16 units with one split are already written
  const bool many = pl.nsplit > 32;
  return launch_combine(out, p, seqlens, H, K, S_max, G, pl.chunk, pl.nsplit, skip_single, d, dtype, many,
                        (long long)B * H, st);
}

}  // namespace

extern "C" {

int gqa_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos, int B,
                  int K, int S_max, int d, gqa_dtype dtype, gqa_stream_t stream) {
  return kv_append_impl(k_cache, v_cache, k_new, v_new, pos, B, K, S_max, d, dtype, stream, nullptr);
}

int gqa_kv_append_paged(void* k_pool, void* v_pool, const void* k_new, const void* v_new, const int32_t* block_table,
                        const int32_t* pos, int B, int K, int d, int num_blocks, int block_size, int max_blocks,
                        gqa_dtype dtype, gqa_stream_t stream) {
  PagedCache pc;
  pc.table = block_table;
  pc.num_blocks = num_blocks;
  pc.block_size = block_size;
  pc.max_blocks = max_blocks;
  if (B < 0 || K <= 0) return GQA_ERR_INVALID_ARG;
  if (!valid_paged(pc, B, K)) return GQA_ERR_SHAPE;
  if (B > 0 && !block_table) return GQA_ERR_INVALID_ARG;
  return kv_append_impl(k_pool, v_pool, k_new, v_new, pos, B, K, max_blocks * block_size, d, dtype, stream, &pc);
}

int gqa_decode(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, int B,
               int H, int K, int S_max, int d, float scale, int num_splits, void* workspace, size_t workspace_bytes,
               gqa_dtype dtype, gqa_stream_t stream) {
  return decode_impl(out, q, k_cache, v_cache, seqlens, B, H, K, S_max, d, scale, num_splits, workspace,
                     workspace_bytes, dtype, stream, nullptr, nullptr, 0);
}

int gqa_decode_append(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                      const int32_t* pos, int B, int H, int K, int S_max, int d, float scale, int num_splits,
                      void* workspace, size_t workspace_bytes, gqa_dtype dtype, gqa_stream_t stream) {
  return decode_impl(out, q, k_cache, v_cache, pos, B, H, K, S_max, d, scale, num_splits, workspace, workspace_bytes,
                     dtype, stream, k_new, v_new, 1);
}

int gqa_decode_paged(void* out, const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                     const int32_t* seqlens, int B, int H, int K, int d, int num_blocks, int block_size,
                     int max_blocks, float scale, int num_splits, void* workspace, size_t workspace_bytes,
                     gqa_dtype dtype, gqa_stream_t stream) {
  PagedCache pc;
  pc.table = block_table;
  pc.num_blocks = num_blocks;
  pc.block_size = block_size;
  pc.max_blocks = max_blocks;
  if (block_size <= 0 || max_blocks <= 0 || (long long)max_blocks * block_size >= (1ll << 31)) return GQA_ERR_SHAPE;
  return decode_impl(out, q, k_pool, v_pool, seqlens, B, H, K, max_blocks * block_size, d, scale, num_splits,
                     workspace, workspace_bytes, dtype, stream, nullptr, nullptr, 0, &pc);
}

int gqa_decode_append_paged(void* out, const void* q, void* k_pool, void* v_pool, const void* k_new,
                            const void* v_new, const int32_t* block_table, const int32_t* pos, int B, int H, int K,
                            int d, int num_blocks, int block_size, int max_blocks, float scale, int num_splits,
                            void* workspace, size_t workspace_bytes, gqa_dtype dtype, gqa_stream_t stream) {
  PagedCache pc;
  pc.table = block_table;
  pc.num_blocks = num_blocks;
  pc.block_size = block_size;
  pc.max_blocks = max_blocks;
  if (block_size <= 0 || max_blocks <= 0 || (long long)max_blocks * block_size >= (1ll << 31)) return GQA_ERR_SHAPE;
  return decode_impl(out, q, k_pool, v_pool, pos, B, H, K, max_blocks * block_size, d, scale, num_splits, workspace,
                     workspace_bytes, dtype, stream, k_new, v_new, 1, &pc);
}

int gqa_decode_int8(void* out, const void* q, const int8_t* k_codes, const float* k_scales, const int8_t* v_codes,
                    const float* v_scales, const int32_t* seqlens, int B, int H, int K, int S_max, int d, float scale,
                    int num_splits, void* workspace, size_t workspace_bytes, gqa_stream_t stream) {
  if (!k_scales || !v_scales) return B == 0 ? GQA_OK : GQA_ERR_INVALID_ARG;
  return decode_impl(out, q, k_codes, v_codes, seqlens, B, H, K, S_max, d, scale, num_splits, workspace,
                     workspace_bytes, GQA_BF16, stream, nullptr, nullptr, 0, nullptr, k_scales, v_scales);
}

size_t gqa_decode_int8_workspace_bytes(int B, int H, int K, int S_max, int d, int num_splits) {
  if (!valid_decode_shape(B, H, K, S_max, d) || d != 128 || S_max % 4 != 0 || num_splits < 0) return 0;
  const DecodePlan a = plan_decode(B, H, K, S_max, d, num_splits, GQA_BF16, sm_count(current_device()), true);
  if (a.ws_bytes == (size_t)-1) return 0;
  return a.ws_bytes;
}

int gqa_kv_append_int8(int8_t* k_codes, float* k_scales, int8_t* v_codes, float* v_scales, const void* k_new,
                       const void* v_new, const int32_t* pos, int B, int K, int S_max, int d, gqa_stream_t stream) {
  if (B < 0 || K <= 0 || S_max <= 0) return GQA_ERR_INVALID_ARG;
  if (d != 128) return GQA_ERR_UNSUPPORTED;
  if (B == 0) return GQA_OK;
  if (!k_codes || !k_scales || !v_codes || !v_scales || !k_new || !v_new || !pos) return GQA_ERR_INVALID_ARG;
  if (!aligned16(k_codes) || !aligned16(v_codes) || !aligned16(k_new) || !aligned16(v_new)) return GQA_ERR_ALIGN;
  const long long warps = 2ll * B * K;
  const int dev = current_device();
  const int grid = grid_for(warps * 32, 256, sm_count(dev));
  return gqa::launch_kernel(gqa::kv_append_int8_kernel, (unsigned)grid, 256, 0, (cudaStream_t)stream, false, k_codes,
                            k_scales, v_codes, v_scales, static_cast<const __nv_bfloat16*>(k_new),
                            static_cast<const __nv_bfloat16*>(v_new), pos, B, K, S_max);
}

size_t gqa_kv_project_workspace_bytes(int B, int T, int K, int d, int d_model) {
  if (!valid_proj(B, T, K, 1, d, d_model)) return 0;
  return plan_proj((long long)B * T, K, d, d_model, sm_count(current_device())).ws_bytes;
}

int gqa_kv_project_append(void* k_cache, void* v_cache, const void* x, const void* w_kv, const int32_t* pos, int B,
                          int T, int K, int S_max, int d, int d_model, void* workspace, size_t workspace_bytes,
                          gqa_dtype dtype, gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (B < 0 || T <= 0 || K <= 0 || S_max <= 0 || d_model <= 0) return GQA_ERR_INVALID_ARG;
  if (!valid_proj(B, T, K, S_max, d, d_model)) return GQA_ERR_SHAPE;
  if (dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if (B == 0) return GQA_OK;
  if (!k_cache || !v_cache || !x || !w_kv) return GQA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(x) || !aligned16(w_kv)) return GQA_ERR_ALIGN;
  const int sms = sm_count(current_device());
  const ProjPlan pl = plan_proj((long long)B * T, K, d, d_model, sms);
  if (pl.ws_bytes > 0 && (!workspace || workspace_bytes < pl.ws_bytes)) return GQA_ERR_INVALID_ARG;
  if (pl.ws_bytes > 0 && !aligned16(workspace)) return GQA_ERR_ALIGN;
  gqa::ProjParams p;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.w = w_kv;
  p.pos = pos;
  p.ws = static_cast<float*>(workspace);
  p.B = B;
  p.T = T;
  p.K = K;
  p.S_max = S_max;
  p.M = B * T;
  p.splits = pl.splits;
  p.ksteps_per_split = d_model / gqa::kPjBK / pl.splits;
  cudaStream_t st = (cudaStream_t)stream;
  return d == 128 ? launch_proj_d<128>(pl, p, x, w_kv, d_model, st, sms)
                  : launch_proj_d<64>(pl, p, x, w_kv, d_model, st, sms);
}

size_t gqa_decode_paged_workspace_bytes(int B, int H, int K, int d, int block_size, int max_blocks, int num_splits) {
  if (block_size <= 0 || block_size % 16 != 0 || max_blocks <= 0 ||
      (long long)max_blocks * block_size >= (1ll << 31))
    return 0;
  const int S_max = max_blocks * block_size;
  if (!valid_decode_shape(B, H, K, S_max, d, true) || num_splits < 0) return 0;
  const DecodePlan a = plan_decode(B, H, K, S_max, d, num_splits, GQA_BF16, sm_count(current_device()), false, true);
  if (a.ws_bytes == (size_t)-1) return 0;
  return a.ws_bytes;
}

int gqa_prefill_causal(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache, int B,
                       int S, int H, int K, int S_max, int d, float scale, gqa_dtype dtype, gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (B < 0 || S < 0 || H <= 0 || K <= 0) return GQA_ERR_INVALID_ARG;
  if (H % K != 0 || (d != 64 && d != 128)) return GQA_ERR_SHAPE;
  if ((k_cache == nullptr) != (v_cache == nullptr)) return GQA_ERR_INVALID_ARG;
  if (k_cache && S > S_max) return GQA_ERR_SHAPE;
  if (B == 0 || S == 0) return GQA_OK;
  if (!out || !q || !k || !v) return GQA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return GQA_ERR_ALIGN;
  if (k_cache && (!aligned16(k_cache) || !aligned16(v_cache))) return GQA_ERR_ALIGN;
  if (dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  return launch_prefill(out, q, k, v, k_cache, v_cache, B, S, H, K, S_max, d, scale, (cudaStream_t)stream,
                        sm_count(current_device()));
}

int gqa_prefill_causal_varlen(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache,
                              const int32_t* cu_seqlens, int B, int T, int H, int K, int S_max, int d, float scale,
                              gqa_dtype dtype, gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H <= 0 || K <= 0) return GQA_ERR_INVALID_ARG;
  if (H % K != 0 || (d != 64 && d != 128)) return GQA_ERR_SHAPE;
  if (dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if ((k_cache == nullptr) != (v_cache == nullptr)) return GQA_ERR_INVALID_ARG;
  if (k_cache && S_max <= 0) return GQA_ERR_INVALID_ARG;
  if ((long long)T + 128ll * (B + 1) >= (1ll << 31)) return GQA_ERR_SHAPE;  // TMA row coordinates are int32
  if (((long long)T / 128 + B + 1) * H >= (1ll << 31)) return GQA_ERR_SHAPE;
  if (B == 0 || T == 0) return GQA_OK;
  if (!out || !q || !k || !v || !cu_seqlens) return GQA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return GQA_ERR_ALIGN;
  if (k_cache && (!aligned16(k_cache) || !aligned16(v_cache))) return GQA_ERR_ALIGN;
  return launch_prefill_varlen(out, q, k, v, k_cache, v_cache, cu_seqlens, B, T, H, K, S_max, d, scale,
                               (cudaStream_t)stream, sm_count(current_device()));
}

int gqa_meanpool_kv(void* dst, const void* src, int64_t outer, int H, int K, int64_t inner, gqa_dtype dtype,
                    gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (outer < 0 || inner < 0 || H <= 0 || K <= 0) return GQA_ERR_INVALID_ARG;
  if (H % K != 0) return GQA_ERR_SHAPE;
  if (outer == 0 || inner == 0) return GQA_OK;
  if (!dst || !src) return GQA_ERR_INVALID_ARG;
  const int elt = dtype == GQA_F32 ? 4 : 2;
  const int vec = 16 / elt;
  const int sms = sm_count(current_device());
  cudaStream_t st = (cudaStream_t)stream;
  if (inner % vec == 0 && aligned16(dst) && aligned16(src)) {
    const long long work = outer * K * (inner / vec);
    const int grid = grid_for(work, 256, sms);
    return gqa::launch_kernel(dtype == GQA_BF16 ? gqa::meanpool_vec_kernel<__nv_bfloat16> : gqa::meanpool_vec_kernel<float>,
                              (unsigned)grid, 256, 0, st, false, static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                              outer, H, K, inner / vec);
  } else {
    if ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & (uintptr_t)(elt - 1))
      return GQA_ERR_ALIGN;
    const long long work = outer * K * inner;
    const int grid = grid_for(work, 256, sms);
    if (dtype == GQA_BF16)
      return gqa::launch_kernel(gqa::meanpool_scalar_kernel<__nv_bfloat16>, (unsigned)grid, 256, 0, st, false,
                                static_cast<__nv_bfloat16*>(dst), static_cast<const __nv_bfloat16*>(src), outer, H, K,
                                inner);
    return gqa::launch_kernel(gqa::meanpool_scalar_kernel<float>, (unsigned)grid, 256, 0, st, false,
                              static_cast<float*>(dst), static_cast<const float*>(src), outer, H, K, inner);
  }
}

int gqa_get_last_error(gqa_stream_t stream, uint32_t* bits) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GQA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, gqa::g_error_word, sizeof(v)) != cudaSuccess) return GQA_ERR_CUDA;
  if (v) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(gqa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return GQA_ERR_CUDA;
  }
  if (bits) *bits = v;
  return v ? GQA_ERR_DEVICE : GQA_OK;
}

}  // extern "C"
