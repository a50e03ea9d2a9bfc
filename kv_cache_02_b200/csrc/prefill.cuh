// Causal GQA prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   out[b, i, h, :] = sum_{j <= i} softmax_j(scale * q[b,i,h] . k[b,j,g]) v[b,j,g],  g = h / (H/K)
//
// One CTA computes one 128-row query tile of one head (two CTAs share an SM:
// 112 KB of shared memory and 256 TMEM columns each). Warp roles:
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r)
//   warp 4     TMA producer: Q once, then 64-key K/V tiles into a 2-stage ring
//   warp 5     MMA issuer (one thread) and TMEM allocator
// Per key tile j:
//   S_j = Q K_j^T   tcgen05.mma, M=128 N=64 K=d, fp32 in TMEM (two S buffers)
//   softmax thread r: tcgen05.ld its S row, causal mask, running max m and sum
//       l in log2 units, P = 2^(S - m) as bf16 into shared memory (128-byte
//       swizzled, the K-major operand layout)
//   O += P V_j      tcgen05.mma, M=128 N=d K=64, fp32 accumulator in TMEM
// The accumulator is rescaled only when a row's maximum grows by more than
// 2^8 (until then P <= 256, exact enough in fp32 and bf16), so most tiles
// touch O only through the MMA. The final O / l is written as bf16.
//
// Heads of one group run in adjacent CTAs, so a K/V tile read from HBM is
// reused from L2 by the group's query heads; the heavy (late) query tiles are
// scheduled first.
#pragma once

#include <atomic>

#include "common.cuh"
#include "tcgen05.cuh"

namespace gqa {

// Three-input maximum, and two fp32 lanes per instruction (Blackwell's
// paired FMA and add): the softmax's per-score arithmetic in half the
// instructions.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (d0, d1) = (a0, a1) * (b, b) + (c, c), each lane rounded once
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %4};\n"
      " mov.b64 rc, {%5, %5};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (s0, s1) += (a0, a1)
__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n .reg .b64 rs, ra;\n mov.b64 rs, {%0, %1};\n mov.b64 ra, {%2, %3};\n"
      " add.rn.f32x2 rs, rs, ra;\n mov.b64 {%0, %1}, rs;\n}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

// Maximum of 64 values as a tree of three-input maxima (depth 4)
__device__ __forceinline__ float max64(const float (&x)[64]) {
  float t[22], u[8];
#pragma unroll
  for (int i = 0; i < 21; ++i) t[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
  t[21] = x[63];
#pragma unroll
  for (int i = 0; i < 7; ++i) u[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  u[7] = t[21];
  return fmax3(fmax3(u[0], u[1], u[2]), fmax3(u[3], u[4], u[5]), fmaxf(u[6], u[7]));
}

constexpr int kPfBM = 128;  // query rows per CTA
constexpr int kPfBN = 64;   // keys per tile
constexpr int kPfStages = 2;
constexpr int kPfThreads = 192;
constexpr int kPfTmemCols = 256;

template <int D>
struct PfCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kQHalf = kPfBM * 128;         // bytes of one 64-column half of Q
  static constexpr int kKVHalf = kPfBN * 128;        // bytes of one 64-column half of a K or V tile
  static constexpr int kQBytes = kHalves * kQHalf;
  static constexpr int kTileBytes = kHalves * kKVHalf;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K and V
  static constexpr int kPBytes = kPfBM * kPfBN * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQBytes;
  static constexpr int kPOff = kKVOff + kPfStages * kStageBytes;
  static constexpr int kBarOff = kPOff + kPBytes;
  static constexpr int kNumBars = 1 + 4 * kPfStages + 2 + 2 + 1 + 1 + 1;
  // at most two CTAs per SM (their 2 x 256 TMEM columns fill the SM's 512)
  static constexpr int kSmemBytes = (kBarOff + kNumBars * 8 + 32) > 80 * 1024 ? (kBarOff + kNumBars * 8 + 32)
                                                                               : 80 * 1024;
  static constexpr int kOCol = 2 * kPfBN;  // TMEM column of O (after the two S buffers)
  static_assert(kOCol + D <= kPfTmemCols, "TMEM budget");
};

struct PrefillParams {
  void* out;  // [B, S, H, D] bf16, or packed [T, H, D] with cu_seqlens
  int B, S, H, K, G, n_qt;
  float scale_log2;
  // varlen (a packed continuous batch): sequence b is tokens cu_seqlens[b] ..
  // cu_seqlens[b+1]-1 of the T rows; null for the fixed-length [B, S] layout
  const int32_t* cu_seqlens;
  int T;
};

template <int D>
__global__ void __launch_bounds__(kPfThreads, 2)
    prefill_causal_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PfCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;                  // TMA Q landed
  uint64_t* k_full = bars + 1;              // [2] TMA K tile landed
  uint64_t* k_empty = k_full + kPfStages;   // [2] S of that tile finished
  uint64_t* v_full = k_empty + kPfStages;   // [2] TMA V tile landed
  uint64_t* v_empty = v_full + kPfStages;   // [2] PV of that tile finished
  uint64_t* s_full = v_empty + kPfStages;   // [2] S buffer written by the MMA
  uint64_t* s_free = s_full + 2;            // [2] S buffer read by all softmax threads
  uint64_t* p_full = s_free + 2;            // P in smem (and O rescaled) for the next PV
  uint64_t* pv_done = p_full + 1;           // the last issued PV finished
  uint64_t* mma_done = pv_done + 1;         // every MMA of this CTA finished
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the 128-byte swizzle pattern assumes 1024-byte aligned operand tiles
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }

  // work item (query tile qt of sequence b, head h): rows seq0 .. seq0+len-1.
  // Fixed length: heavy query tiles first, the G heads of a group adjacent.
  // Varlen: tiles sequence by sequence, each sequence's heaviest first, the
  // heads of a tile adjacent; thread 0 finds the tile's sequence (the grid is
  // sized for the worst case, and CTAs past the last tile end here).
  int qt, b, h, seq0, len;
  if (p.cu_seqlens == nullptr) {
    const int per_qt = p.B * p.H;
    qt = p.n_qt - 1 - (int)(blockIdx.x / per_qt);
    const int rem = (int)(blockIdx.x % per_qt);
    b = rem / p.H;
    h = rem % p.H;
    seq0 = b * p.S;
    len = p.S;
  } else {
    int* s_item = reinterpret_cast<int*>(smem + C::kBarOff + C::kNumBars * 8 + 8);
    h = (int)(blockIdx.x % p.H);
    const int t_idx = (int)(blockIdx.x / p.H);
    if (threadIdx.x == 0) {
      // sequence by sequence, each sequence's heaviest tile first (measured
      // faster than ordering all sequences' tiles by weight: a sequence's K/V
      // tiles stay hot in L2 while its query tiles run)
      int acc = 0, fb = -1, fs0 = 0, flen = 0, fqt = 0;
      bool bad = false;
      for (int bb = 0; bb < p.B; ++bb) {
        int s0 = __ldg(p.cu_seqlens + bb), s1 = __ldg(p.cu_seqlens + bb + 1);
        if (s0 < 0 || s1 > p.T || s1 < s0) bad = true;  // clamped to the packed rows
        s0 = min(max(s0, 0), p.T);
        s1 = min(max(s1, s0), p.T);
        const int n = (s1 - s0 + kPfBM - 1) / kPfBM;
        if (fb < 0 && t_idx < acc + n) {
          fb = bb;
          fs0 = s0;
          flen = s1 - s0;
          fqt = n - 1 - (t_idx - acc);
        }
        acc += n;
      }
      if (bad && blockIdx.x == 0) raise_error(GQA_DEVERR_SEQLEN);
      s_item[0] = fb;
      s_item[1] = fs0;
      s_item[2] = flen;
      s_item[3] = fqt;
    }
    __syncthreads();
    b = s_item[0];
    seq0 = s_item[1];
    len = s_item[2];
    qt = s_item[3];
    if (b < 0) return;
  }
  const int g = h / p.G;
  const int q0 = qt * kPfBM;
  const int n_tiles = min((len + kPfBN - 1) / kPfBN, (q0 + kPfBM + kPfBN - 1) / kPfBN);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // -------------------------------------------------------------- TMA
    // lane 0 loads Q and the K tiles, lane 1 the V tiles: a K stage is free
    // again as soon as its S is computed, a V stage only after its PV
    if (lane < 2) {
      const bool is_k = lane == 0;
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const int buf_off = C::kKVOff + (is_k ? 0 : C::kTileBytes);
      prefetch_tensormap(tm);
      const uint64_t pol_kv = l2_policy_evict_last();
      if (is_k) {
        prefetch_tensormap(&tm_q);
        const uint64_t pol_q = l2_policy_evict_first();
        mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_3d(smem + C::kQOff + hf * C::kQHalf, &tm_q, hf * 64, h, seq0 + q0, q_full, pol_q);
      }
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kPfStages;
        if (j >= kPfStages && !mbar_wait_bounded(&empty[s], ((j / kPfStages) - 1) & 1)) break;
        uint8_t* dst = smem + buf_off + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_3d(dst + hf * C::kKVHalf, tm, hf * 64, g, seq0 + j * kPfBN, &full[s], pol_kv);
        ++issued;
      }
      for (int j = max(0, issued - kPfStages); j < issued; ++j)
        mbar_wait_bounded(&full[j % kPfStages], (j / kPfStages) & 1);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA
    // The warp runs converged (descriptors are warp-uniform values) and one
    // elected lane issues each tcgen05 instruction.
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_bf16_f32(kPfBM, kPfBN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kPfBM, D, false, true);
    const uint32_t q_addr = smem_u32(smem + C::kQOff);
    const uint32_t p_addr = smem_u32(smem + C::kPOff);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    bool ok = wait_all(q_full, 0);
    auto issue_s = [&](int j) -> bool {
      const int s = j % kPfStages;
      if (!wait_all(&k_full[s], (j / kPfStages) & 1)) return false;
      if (j >= 2 && !wait_all(&s_free[j & 1], ((j >> 1) - 1) & 1)) return false;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(smem + C::kKVOff + s * C::kStageBytes);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 columns = 32 bytes inside the 128-byte swizzle row
          const uint64_t ad = smem_desc_sw128(q_addr + (kk >> 2) * C::kQHalf + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + (kk >> 2) * C::kKVHalf + off, 16, 1024);
          tc_mma(tmem + (uint32_t)((j & 1) * kPfBN), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
      commit(&s_full[j & 1]);
      commit(&k_empty[s]);
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; ok && j < n_tiles; ++j) {
      if (j + 1 < n_tiles && !issue_s(j + 1)) {
        ok = false;
        break;
      }
      if (!wait_all(p_full, j & 1) || !wait_all(&v_full[j % kPfStages], (j / kPfStages) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t v_addr = smem_u32(smem + C::kKVOff + (j % kPfStages) * C::kStageBytes + C::kTileBytes);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(p_addr + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v_addr + kk * 16 * 128, C::kKVHalf, 1024);
          tc_mma(tmem + C::kOCol, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
      commit(pv_done);
      commit(&v_empty[j % kPfStages]);
    }
    commit(mma_done);
    wait_all(mma_done, 0);
  } else {
    // ---------------------------------------------------------- softmax
    const int r = threadIdx.x;  // query row within the tile = TMEM lane
    const int qpos = q0 + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* prow = smem + C::kPOff + r * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      // tcgen05.ld/st are warp-collective: every decision that guards them is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[64];
      {
        float a[32], c[32];
        tmem_ld32(lane_addr + (uint32_t)((j & 1) * kPfBN), a);
        tmem_ld32(lane_addr + (uint32_t)((j & 1) * kPfBN + 32), c);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = a[i];
          x[32 + i] = c[i];
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[j & 1]);

      const int k0 = j * kPfBN;
      const int kmax = min(qpos, len - 1) - k0;  // keys k0 + c with c <= kmax are visible
      // With a positive scale the maximum is taken on the raw scores and the
      // scale folds into the exponent (one FFMA per score); off-diagonal
      // tiles need no mask.
      const float sl2 = p.scale_log2;
      const bool pos_scale = sl2 > 0.f;  // the same in every thread
      if (!(pos_scale && kmax >= kPfBN - 1)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = c <= kmax ? (pos_scale ? x[c] : x[c] * sl2) : -INFINITY;
      }
      float mt = max64(x);
      const float xs = pos_scale ? sl2 : 1.f;  // scale still to apply to x
      mt *= xs;
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_used + 8.f) {  // first tile: m_used = -inf
        const float m_new = fmaxf(mt, m_used);
        alpha = fast_exp2(m_used - m_new);
        rescale = j > 0;
        m_used = m_new;
      }
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;  // four partial sums, two per paired add
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float y0, y1;
        fma2(y0, y1, x[2 * c], x[2 * c + 1], xs, -m_used);
        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
        if (c & 1)
          add2(s2, s3, p0, p1);
        else
          add2(s0, s1, p0, p1);
        pk[c] = pack_bf16x2(p0, p1);
      }
      const float sum = (s0 + s1) + (s2 + s3);
      l = l * alpha + sum;
      // P buffer and O are free once the previous tile's PV has finished
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (j - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {  // lanes that keep their max scale by alpha = 1
#pragma unroll 1
        for (int cb = 0; cb < D; cb += 32) {
          float o[32];
          tmem_ld32(lane_addr + C::kOCol + cb, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(lane_addr + C::kOCol + cb, o);
        }
        tc_wait_st();
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = ((uint32_t)(c ^ (r & 7))) << 4;
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue: O / l -> bf16
    if (__all_sync(0xffffffffu, ok && mbar_wait_bounded(pv_done, (n_tiles - 1) & 1))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      // 64 columns at a time; the row's eight 16-byte pieces are transposed across each group
      // of 8 lanes (butterfly shuffles) so that each store instruction writes 4 rows x 128
      // contiguous bytes instead of a 16-byte piece of 32 rows
      const int j = lane & 7;
#pragma unroll 1
      for (int cb = 0; cb < D; cb += 64) {
        float o[64];
        tmem_ld32(lane_addr + C::kOCol + cb, *reinterpret_cast<float(*)[32]>(&o[0]));
        tmem_ld32(lane_addr + C::kOCol + cb + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
        tc_wait_ld();
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
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
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int qk = __shfl_sync(0xffffffffu, qpos, (lane & ~7) + k);  // row k of the group
          if (qk < len)
            reinterpret_cast<uint4*>(out + (((size_t)seq0 + qk) * p.H + h) * D + cb)[j] =
                make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
        __syncwarp();  // converged again for the next warp-collective TMEM loads
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host launch

typedef CUresult (*PfEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [B*S, heads, D] bf16 viewed as (x = D, y = heads, z = B*S); box 64 x 1 x rows
inline bool encode_bsh(PfEncodeFn fn, CUtensorMap* map, const void* base, uint64_t BS, uint64_t heads, uint64_t Dd,
                       uint32_t rows) {
  cuuint64_t dims[3] = {Dd, heads, BS};
  cuuint64_t strides[2] = {Dd * 2, heads * Dd * 2};
  cuuint32_t box[3] = {64, 1, rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Fixed length: q/out [B, S, H, D], k/v [B, S, K, D] (cu_seqlens null).
// Varlen: packed q/out [T, H, D], k/v [T, K, D], B sequences given by
// cu_seqlens (device); S is unused and the grid covers the worst case of
// ceil(T / 128) + B query tiles per head.
template <int D>
int launch_prefill_d(PfEncodeFn fn, void* out, const void* q, const void* k, const void* v, int B, int S, int H,
                     int K, float scale, cudaStream_t st, const int32_t* cu_seqlens = nullptr, int T = 0) {
  using C = PfCfg<D>;
  CUtensorMap tq, tk, tv;
  const uint64_t rows = cu_seqlens ? (uint64_t)T : (uint64_t)B * S;
  if (!encode_bsh(fn, &tq, q, rows, H, D, kPfBM) || !encode_bsh(fn, &tk, k, rows, K, D, kPfBN) ||
      !encode_bsh(fn, &tv, v, rows, K, D, kPfBN))
    return GQA_ERR_CUDA;
  // once per device; concurrent host threads may both set it (same value)
  static std::atomic<int> configured[64]{};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  if (dev >= 0 && dev < 64 && configured[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(prefill_causal_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return GQA_ERR_CUDA;
    configured[dev].store(1, std::memory_order_release);
  }
  PrefillParams p;
  p.out = out;
  p.B = B;
  p.S = S;
  p.H = H;
  p.K = K;
  p.G = H / K;
  p.n_qt = (S + kPfBM - 1) / kPfBM;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cu_seqlens = cu_seqlens;
  p.T = T;
  const long long grid = cu_seqlens ? ((long long)(T + kPfBM - 1) / kPfBM + B) * H : (long long)p.n_qt * B * H;
  return launch_kernel(prefill_causal_kernel<D>, (unsigned)grid, kPfThreads, C::kSmemBytes, st, false, tq, tk, tv, p);
}

}  // namespace gqa
