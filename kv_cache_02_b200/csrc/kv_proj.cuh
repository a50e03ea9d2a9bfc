// Fused K/V projection into the cache on the 5th-generation tensor cores.
//
//   [K_g | V_g](token) = W_KV[g] x(token),  W_KV: [K, 2D, d_model], x: [tokens, d_model]
//
// ("GQA 完全拆解", section 工程实现：权重布局、repeat 与 Kernel 融合: engines merge
// W_K and W_V into one W_KV so that one GEMM yields K and V.) The rows go
// straight into the cache at the token's key: token i of sequence b at key
// pos[b] + i.
//
// One CTA computes a 128-token x 2D-output tile (all of one KV head's K and
// V) over a range of d_model: tcgen05.mma M=128 N=2D K=16, both operands
// K-major with the 128-byte swizzle, fed by TMA through a 4-stage ring, the
// fp32 accumulator in TMEM (lane = token row). Warp roles: 0-3 epilogue,
// 4 TMA producer, 5 TMEM allocation and the MMA-issuing thread.
//
// When the token tiles and heads alone would leave SMs idle, d_model is
// split over CTAs: each split writes its fp32 partial tile to a workspace
// slice of its own (no atomics, nothing to zero) and kv_proj_finalize_kernel
// sums the splits and writes the rows. A decode step (a few tokens) uses
// kv_proj_small_kernel, with the operands swapped.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace gqa {

constexpr int kPjBM = 128;  // tokens per CTA
constexpr int kPjBK = 64;   // d_model per stage (one 128-byte swizzle row of bf16)
constexpr int kPjStages = 4;
constexpr int kPjThreads = 192;

template <int D>
struct PjCfg {
  static constexpr int kN = 2 * D;                    // outputs per CTA: K then V of one head
  static constexpr int kABytes = kPjBM * kPjBK * 2;    // 16 KB
  static constexpr int kBBytes = kN * kPjBK * 2;       // 32 KB (D = 128)
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOff = kPjStages * kStageBytes;
  static constexpr int kNumBars = 2 * kPjStages + 1;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kTmemCols = kN;                 // fp32 accumulator columns
};

struct ProjParams {
  void* k_cache;         // [B, K, S_max, D] bf16
  void* v_cache;
  const int32_t* pos;    // [B]: key of each sequence's first new token, or null (0)
  float* ws;             // splits > 1: partials [splits][M][K * 2D] fp32
  int B, T, K, S_max, M, ksteps_per_split, splits;
};

// Token m of the batch: sequence m / T, new token m % T, written at key
// pos[b] + m % T; a sequence whose rows do not fit sets GQA_DEVERR_APPEND_POS
// (reported by its first token for head 0) and is not written.
__device__ __forceinline__ bool proj_row(const ProjParams& p, int m, int g, size_t& row) {
  const int b = m / p.T, i = m % p.T;
  const int p0 = p.pos ? __ldg(p.pos + b) : 0;
  if (p0 < 0 || p0 > p.S_max - p.T) {
    if (i == 0 && g == 0) raise_error(GQA_DEVERR_APPEND_POS);
    return false;
  }
  row = ((size_t)b * p.K + g) * p.S_max + p0 + i;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kPjThreads, 1)
    kv_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const ProjParams p) {
  using C = PjCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;                  // [stages] x and W tiles landed
  uint64_t* empty = bars + kPjStages;     // [stages] the MMAs reading them finished
  uint64_t* acc_full = empty + kPjStages; // every MMA of this CTA finished
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (smem_u32(smem) & 1023u) {  // the swizzle pattern needs 1024-byte aligned tiles
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  // tile: token tile mt, head g, d_model split sp
  const int per_mt = p.K * p.splits;
  const int mt = (int)(blockIdx.x / per_mt);
  const int g = (int)(blockIdx.x % per_mt) / p.splits;
  const int sp = (int)(blockIdx.x % p.splits);
  const int k_begin = sp * p.ksteps_per_split;
  const int nk = p.ksteps_per_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the finalize pass may be scheduled

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_w);
      const uint64_t pol_x = l2_policy_evict_last();   // a token tile is read by every head
      const uint64_t pol_w = l2_policy_evict_first();  // W is streamed
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % kPjStages;
        if (j >= kPjStages && !mbar_wait_bounded(&empty[s], ((j / kPjStages) - 1) & 1)) break;
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)C::kStageBytes);
        const int kx = (k_begin + j) * kPjBK;
        tma_load_2d(st, &tm_x, kx, mt * kPjBM, &full[s], pol_x);
        tma_load_2d(st + C::kABytes, &tm_w, kx, g * C::kN, &full[s], pol_w);
        ++issued;
      }
      for (int j = max(0, issued - kPjStages); j < issued; ++j) mbar_wait_bounded(&full[j % kPjStages], (j / kPjStages) & 1);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPjBM, C::kN, false, false);
      bool ok = true;
      for (int j = 0; j < nk && ok; ++j) {
        const int s = j % kPjStages;
        if (!(ok = mbar_wait_bounded(&full[s], (j / kPjStages) & 1))) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes);
        const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
        for (int kk = 0; kk < kPjBK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          tc_mma(tmem, ad, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);  // completes when every MMA issued above has finished
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int r = threadIdx.x;  // token row within the tile = TMEM lane
    const int m = mt * kPjBM + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    if (__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, 0))) {
      tc_fence_after();
      size_t row = 0;
      const bool valid = m < p.M && (p.splits > 1 || proj_row(p, m, g, row));
#pragma unroll 1
      for (int cb = 0; cb < C::kN; cb += 32) {
        float o[32];
        tmem_ld32(lane_addr + cb, o);  // warp-collective: every lane takes part
        tc_wait_ld();
        if (!valid) continue;
        if (p.splits > 1) {
          float4* dst = reinterpret_cast<float4*>(p.ws + ((size_t)sp * p.M + m) * ((size_t)p.K * C::kN) +
                                                  (size_t)g * C::kN + cb);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        } else {
          __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(cb < D ? p.k_cache : p.v_cache);
          uint4* dst = reinterpret_cast<uint4*>(cache + row * D + (cb % D));
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(o[8 * i], o[8 * i + 1]), pack_bf16x2(o[8 * i + 2], o[8 * i + 3]),
                                pack_bf16x2(o[8 * i + 4], o[8 * i + 5]), pack_bf16x2(o[8 * i + 6], o[8 * i + 7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// A decode step (at most kPsTok tokens): the operands swap. A = 128 rows of
// W_KV (outputs), B = the tokens (padded to 16), D = [128 outputs x 16
// tokens] in TMEM (lane = output), so the MMA does 16x less padding work
// than with tokens as M and every CTA streams its own slice of W_KV.
// Epilogue thread r holds output r for every token: across a warp 32
// consecutive outputs of one token, 64 contiguous bytes of a cache row.
constexpr int kPsRows = 128;  // W_KV rows (outputs) per CTA
constexpr int kPsTok = 16;    // tokens (MMA N)

struct PsCfg {
  static constexpr int kABytes = kPsRows * kPjBK * 2;  // 16 KB of W
  static constexpr int kBBytes = kPsTok * kPjBK * 2;   // 2 KB of x
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOff = kPjStages * kStageBytes;
  static constexpr int kNumBars = 2 * kPjStages + 1;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kTmemCols = 32;  // 16 used (the allocation minimum is 32)
};

template <int D>
__global__ void __launch_bounds__(kPjThreads)
    kv_proj_small_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const ProjParams p) {
  using C = PsCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + kPjStages;
  uint64_t* acc_full = empty + kPjStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  const int ft = (int)(blockIdx.x / p.splits);  // tile of 128 W_KV rows
  const int sp = (int)(blockIdx.x % p.splits);
  const int k_begin = sp * p.ksteps_per_split;
  const int nk = p.ksteps_per_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the finalize pass may be scheduled

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_w);
      const uint64_t pol_x = l2_policy_evict_last();
      const uint64_t pol_w = l2_policy_evict_first();
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % kPjStages;
        if (j >= kPjStages && !mbar_wait_bounded(&empty[s], ((j / kPjStages) - 1) & 1)) break;
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)C::kStageBytes);
        const int kx = (k_begin + j) * kPjBK;
        tma_load_2d(st, &tm_w, kx, ft * kPsRows, &full[s], pol_w);
        tma_load_2d(st + C::kABytes, &tm_x, kx, 0, &full[s], pol_x);
        ++issued;
      }
      for (int j = max(0, issued - kPjStages); j < issued; ++j) mbar_wait_bounded(&full[j % kPjStages], (j / kPjStages) & 1);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPsRows, kPsTok, false, false);
      bool ok = true;
      for (int j = 0; j < nk && ok; ++j) {
        const int s = j % kPjStages;
        if (!(ok = mbar_wait_bounded(&full[s], (j / kPjStages) & 1))) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes);
        const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
        for (int kk = 0; kk < kPjBK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          tc_mma(tmem, ad, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);
    }
  } else {
    const int f = ft * kPsRows + threadIdx.x;  // W_KV row: head f / 2D, K (< D) or V, dim f % D
    const int g = f / (2 * D), jd = f % (2 * D);
    if (__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, 0))) {
      tc_fence_after();
      float o[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), o);
      tc_wait_ld();
      const size_t ncols = (size_t)p.K * 2 * D;
#pragma unroll
      for (int t = 0; t < kPsTok; ++t) {
        if (t >= p.M) break;
        if (p.splits > 1) {
          p.ws[((size_t)sp * p.M + t) * ncols + f] = o[t];
        } else {
          size_t row = 0;
          if (!proj_row(p, t, g, row)) continue;
          __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(jd < D ? p.k_cache : p.v_cache);
          cache[row * D + (jd % D)] = __float2bfloat16_rn(o[t]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Split d_model: the sum of the splits' partials, rounded once to bf16 and
// written at the token's key. One thread per output (consecutive outputs in
// consecutive threads); the splits' partials (at most kPjMaxSplits) are all
// loaded before any is summed, one round trip. Launched as a programmatic
// dependent of the GEMM: it waits for that grid before reading.
constexpr int kPjMaxSplits = 16;

template <int D>
__global__ void kv_proj_finalize_kernel(const ProjParams p) {
  constexpr int kN = 2 * D;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t ncols = (size_t)p.K * kN;
  const long long total = (long long)p.M * (long long)ncols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int f = (int)(i % (long long)ncols);
    const int m = (int)(i / (long long)ncols);
    const int g = f / kN, j = f % kN;
    size_t row = 0;
    if (!proj_row(p, m, g, row)) continue;
    float v[kPjMaxSplits];
#pragma unroll
    for (int s = 0; s < kPjMaxSplits; ++s)
      v[s] = s < p.splits ? __ldcg(p.ws + ((size_t)s * p.M + m) * ncols + f) : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int s = 0; s < kPjMaxSplits; ++s) acc += v[s];
    __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(j < D ? p.k_cache : p.v_cache);
    cache[row * D + (j % D)] = __float2bfloat16_rn(acc);
  }
}

}  // namespace gqa
