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
// kv_proj_gemv_kernel, which streams W_KV once with no split.
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
  const void* w;         // W_KV [K * 2D, d_model] bf16 (for the L2 warm-up of a decode step)
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
    // converged warp (warp-uniform descriptors), one elected lane issues
    const bool leader = elect_one();
    constexpr uint32_t idesc = idesc_bf16_f32(kPjBM, C::kN, false, false);
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      const int s = j % kPjStages;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (j / kPjStages) & 1)))) break;
      tc_fence_after();
      const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes);
      const uint32_t b_addr = a_addr + C::kABytes;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kPjBK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          tc_mma(tmem, ad, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (leader) tc_commit(acc_full);  // completes when every MMA issued above has finished
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue
    const int r = threadIdx.x;  // token row within the tile = TMEM lane
    const int m = mt * kPjBM + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    if (__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, 0))) {
      tc_fence_after();
      size_t row = 0;
      const bool valid = m < p.M && (p.splits > 1 || proj_row(p, m, g, row));
      __syncwarp();  // the lanes reconverge before the warp-collective TMEM loads
      if (p.splits > 1) {
#pragma unroll 1
        for (int cb = 0; cb < C::kN; cb += 32) {
          float o[32];
          tmem_ld32(lane_addr + cb, o);  // warp-collective: every lane takes part
          tc_wait_ld();
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(p.ws + ((size_t)sp * p.M + m) * ((size_t)p.K * C::kN) +
                                                    (size_t)g * C::kN + cb);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
          __syncwarp();  // converged again for the next TMEM loads
        }
      } else {
        // 64 columns (a 128-byte segment of a cache row) at a time. Thread r holds token r's
        // row, so a store instruction would write a 16-byte piece of 32 rows; the 8 pieces are
        // transposed across each group of 8 lanes by butterfly shuffles, and store k of lane j
        // writes piece j of the group's row k: 4 whole segments per instruction.
        const int j = lane & 7;
#pragma unroll 1
        for (int cb = 0; cb < C::kN; cb += 64) {
          float o[64];
          tmem_ld32(lane_addr + cb, *reinterpret_cast<float(*)[32]>(&o[0]));
          tmem_ld32(lane_addr + cb + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
          tc_wait_ld();
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
#pragma unroll
          for (int mk = 1; mk < 8; mk <<= 1) {
            const bool up = (j & mk) != 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              if (c & mk) continue;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t send = up ? w[4 * c + e] : w[4 * (c | mk) + e];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, mk);
                if (up)
                  w[4 * c + e] = recv;
                else
                  w[4 * (c | mk) + e] = recv;
              }
            }
          }
          __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(cb < D ? p.k_cache : p.v_cache);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int src = (lane & ~7) + k;  // the lane that holds row k of the group
            const unsigned long long rk = __shfl_sync(0xffffffffu, (unsigned long long)row, src);
            const bool vk = __shfl_sync(0xffffffffu, valid ? 1 : 0, src) != 0;
            if (vk)
              reinterpret_cast<uint4*>(cache + rk * D + (cb % D))[j] =
                  make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
          __syncwarp();  // converged again for the next TMEM loads
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

// A decode step (at most kPsTok = 16 tokens): a weight-streaming GEMV.
// Every W_KV row is read once and multiplied by the few tokens: 2 * tokens
// flop per 2 bytes of W, so HBM bound; the tensor cores are needed only to
// keep up with the stream (fp32 FMA would not), and the warp-level
// mma.sync m16n8k16 fits a 16-row x 8-token tile without padding rows.
//
// One CTA owns 16 consecutive W_KV rows (outputs) over all of d_model, so
// there is no split and nothing to merge across CTAs: no workspace and no
// second pass. Its W slice streams through a ring of kGvStages stages of 512
// columns (16 KB of W with the same columns of x) loaded by TMA; with
// d_model = 4096 the whole 128 KB slice is requested at once. Consumer warp
// w takes the stages w, w + kGvStages, ...: per 16 columns an ldmatrix of W
// (A, 16 rows), an ldmatrix of x (B, 8 tokens) per 8 tokens, one MMA. At the
// end the warps' partial tiles are summed in shared memory and the rows
// written, bf16, at each token's key.
constexpr int kPsTok = 16;    // most tokens of a decode step
constexpr int kGvRows = 16;   // W_KV rows per CTA
constexpr int kGvCols = 512;  // d_model columns per stage (8 blocks of 64)
#ifndef GQA_GV_WARM
#define GQA_GV_WARM 1
#endif
constexpr bool kGvWarm = GQA_GV_WARM != 0;  // L2 warm-up of the W_KV slice before the grid dependency

template <int NT>  // token tiles of 8: 1 (up to 8 tokens) or 2 (up to 16)
struct GvCfg {
  static constexpr int kStages = NT == 1 ? 8 : 6;          // = consumer warps
  static constexpr int kThreads = (kStages + 1) * 32;      // + the TMA producer warp
  static constexpr int kWBytes = kGvRows * kGvCols * 2;    // 16 KB
  static constexpr int kXBytes = 8 * NT * kGvCols * 2;     // 8 KB per token tile
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kRedOff = kStages * kStageBytes;    // [warps][16 rows][8 NT tokens] fp32
  static constexpr int kBarOff = kRedOff + kStages * kGvRows * 8 * NT * 4;
  static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8;
};

// tm_w: W_KV as (64 columns, rows, d_model / 64 blocks), box (64, 16, 8);
// tm_x: x as (64, tokens, d_model / 64), box (64, 8 NT, 8) (token rows past
// the batch read as zeros). Both 128-byte swizzled: in a stage, W block b,
// row r is the 128-byte line b * 16 + r, x block b, token n the line b * 8 NT + n.
template <int D, int NT>
__global__ void __launch_bounds__(GvCfg<NT>::kThreads, 1)
    kv_proj_gemv_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                        const ProjParams p, int d_model) {
  using C = GvCfg<NT>;
  constexpr int kW = C::kStages;  // consumer warps
  extern __shared__ __align__(1024) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + kW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (d_model + kGvCols - 1) / kGvCols;  // stages of the whole row slice
  const int row0 = (int)blockIdx.x * kGvRows;

  if (smem_u32(smem) & 1023u) {
    grid_dep_wait();
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kW; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // W_KV rows are weights: warm L2 with this CTA's slice while the kernel
  // before finishes (a hint; the loads below come after the grid dependency)
  if (kGvWarm && warp == kW && lane < kGvRows)
    for (int c = 0; c < d_model * 2; c += 32768)
      prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(p.w) + ((size_t)(row0 + lane) * d_model) * 2 + c,
                       (uint32_t)min(32768, d_model * 2 - c));
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kW) {
    // ------------------------------------------------------------ producer
    // The first pass over the ring is issued by one lane per stage at once;
    // stages past it (d_model > kW * 512) by lane 0 as consumers free them.
    const uint64_t pol_w = l2_policy_evict_first();  // streamed once
    const uint64_t pol_x = l2_policy_evict_last();   // read by every CTA
    auto issue = [&](int j) {
      const int s = j % kW;
      uint8_t* st = smem + s * C::kStageBytes;
      mbar_arrive_expect_tx(&full[s], (uint32_t)C::kStageBytes);
      tma_load_3d(st, &tm_w, 0, row0, j * (kGvCols / 64), &full[s], pol_w);
      tma_load_3d(st + C::kWBytes, &tm_x, 0, 0, j * (kGvCols / 64), &full[s], pol_x);
    };
    if (lane == 0) {
      prefetch_tensormap(&tm_w);
      prefetch_tensormap(&tm_x);
    }
    __syncwarp();
    if (lane < min(kW, nkb)) issue(lane);
    if (lane == 0) {
      int issued = min(kW, nkb);
      for (int j = kW; j < nkb; ++j) {
        if (!mbar_wait_bounded(&empty[j % kW], ((j / kW) - 1) & 1)) break;
        issue(j);
        ++issued;
      }
      // this CTA's loads land before it may exit (the consumers may have given up)
      for (int j = max(0, issued - kW); j < issued; ++j) mbar_wait_bounded(&full[j % kW], (j / kW) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // ldmatrix rows: A (W) matrices (rows 0-7 | 8-15) x (chunk c | c+1); B (x)
  // matrices (tokens 0-7) x (chunks c, c+1, c+2, c+3): two 16-column steps
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int a_chk = lane >> 4;
  const int b_tok = lane & 7;
  const int b_chk = lane >> 3;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  bool ok = true;
  for (int j = warp, n = 0; j < nkb; j += kW, ++n) {
    if (!(ok = mbar_wait_bounded(&full[warp], n & 1))) break;
    const uint32_t wa = smem_u32(smem + warp * C::kStageBytes);
    const uint32_t xa = wa + C::kWBytes;
#pragma unroll 4
    for (int b = 0; b < kGvCols / 64; ++b) {  // 64-column block: 4 steps of 16 columns
#pragma unroll
      for (int h = 0; h < 2; ++h) {           // two steps at a time: chunks 4h .. 4h + 3
        uint32_t a[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int line = b * kGvRows + a_row;
          const int chk = 4 * h + 2 * u + a_chk;
          ldmatrix_x4(wa + line * 128 + ((chk ^ (line & 7)) << 4), a[u][0], a[u][1], a[u][2], a[u][3]);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int line = b * 8 * NT + 8 * t + b_tok;
          const int chk = 4 * h + b_chk;
          uint32_t x0, x1, x2, x3;
          ldmatrix_x4(xa + line * 128 + ((chk ^ (line & 7)) << 4), x0, x1, x2, x3);
          mma_bf16_16816(acc[t], a[0][0], a[0][1], a[0][2], a[0][3], x0, x1);
          mma_bf16_16816(acc[t], a[1][0], a[1][1], a[1][2], a[1][3], x2, x3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[warp]);
  }
  // the warps' partial [16 rows x 8 NT tokens] tiles: accumulator (row g | g + 8, tokens 2c, 2c + 1)
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float* rw = red + (size_t)warp * kGvRows * 8 * NT;
    rw[g * 8 * NT + 8 * t + 2 * c] = acc[t][0];
    rw[g * 8 * NT + 8 * t + 2 * c + 1] = acc[t][1];
    rw[(g + 8) * 8 * NT + 8 * t + 2 * c] = acc[t][2];
    rw[(g + 8) * 8 * NT + 8 * t + 2 * c + 1] = acc[t][3];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kW * 32) : "memory");  // the consumer warps (the producer has left)
  // output (row r, token m): thread m * 16 + r, 16 rows of a token = 32 contiguous bytes of a cache row
  for (int o = threadIdx.x; o < kGvRows * 8 * NT; o += kW * 32) {
    const int m = o / kGvRows, r = o % kGvRows;
    if (m >= p.M) continue;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) sum += red[((size_t)w * kGvRows + r) * 8 * NT + m];
    const int f = row0 + r;  // W_KV row: head f / 2D, K (< D) or V, dim f % D
    const int gh = f / (2 * D), jd = f % (2 * D);
    size_t crow = 0;
    if (!proj_row(p, m, gh, crow)) continue;
    __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(jd < D ? p.k_cache : p.v_cache);
    cache[crow * D + (jd % D)] = __float2bfloat16_rn(sum);
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
