// GQA decode over a KV cache (split-KV with a log-sum-exp combine).
//
// One CTA owns one work item (b, g, split, head slice): the keys
// [split*chunk, min(len_b, (split+1)*chunk)) of KV head g of sequence b, and up
// to 8 query heads of that group. Every K/V row is brought from HBM once by
// TMA and serves all the CTA's query heads ("GQA 完全拆解", section 工程实现:
// the group's query heads share one thread block and one load of each KV
// block).
//
// bf16 path, per CTA: warp 4 is the TMA producer (64-key tiles of K and V,
// 128-byte swizzled, a ring of mbarrier-guarded stages); warps 0..3 each own
// 16 keys of every tile and run on the tensor cores:
//     S^T[16 keys x 8 heads]  = K[16 x d] * Q^T[d x 8]        (mma.sync m16n8k16)
//     online softmax over keys, per head, in fp32 (log2 domain)
//     O^T[d x 8 heads]       += V^T[d x 16 keys] * P^T[16 x 8]
// Keys sit in the MMA M dimension and the group's heads in N, so G = 8 fills
// the instruction and G = 4 uses half of it. P^T is produced from the S^T
// accumulator with movmatrix (register transpose), with no shared-memory trip.
// The four warps' partial (m, l, O) are merged in shared memory; the CTA then
// writes either the final output (one split) or its partial to the workspace
// for decode_combine_kernel.
//
// f32 path (small problems, float32 storage): plain FMA, one warp per head.
#pragma once

#include "common.cuh"

namespace gqa {

constexpr int kDecTileKeys = 64;
constexpr int kDecConsumerWarps = 4;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecBoxRows = 16;  // TMA box height; the ragged tail is read in 16-row steps
constexpr int kDecHeadsPerCta = 8;

template <int D>
struct DecCfg {
  static constexpr int kHalves = D / 64;                       // 128-byte column boxes per row
  static constexpr int kHalfBytes = kDecTileKeys * 128;        // one column box of a tile
  static constexpr int kTileBytes = kDecTileKeys * D * 2;      // K (or V) tile
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8 + 1024;  // + alignment slack
  static_assert(kDecConsumerWarps * (kDecHeadsPerCta * D + 2 * kDecHeadsPerCta) * 4 <= kBarOffset,
                "merge scratch must fit in the stage buffers");
};

struct DecodeParams {
  const void* q;
  void* out;
  float* ws_o;    // [B*K*nsplit*G, D] partial O (unnormalised, relative to m)
  float2* ws_ml;  // [B*K*nsplit*G] partial (m, l), m in log2 units
  const int32_t* seqlens;
  int B, H, K, S_max, G, hslices, chunk, nsplit;
  float scale_log2;  // scale * log2(e)
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Work item -> (unit, split, head slice); head slice varies fastest so the
// CTAs that read the same KV chunk for different head slices run together.
struct DecItem {
  int b, g, unit, split, hsl, len, t_begin, t_end, h0, nh;
};

__device__ __forceinline__ DecItem decode_item(const DecodeParams& p, int heads_per_cta) {
  DecItem it;
  const int item = blockIdx.x;
  it.hsl = item % p.hslices;
  const int rest = item / p.hslices;
  it.split = rest % p.nsplit;
  it.unit = rest / p.nsplit;
  it.b = it.unit / p.K;
  it.g = it.unit % p.K;
  int len = __ldg(p.seqlens + it.b);
  if (len < 0 || len > p.S_max) {
    if (it.split == 0 && it.hsl == 0 && it.g == 0 && threadIdx.x == 0) raise_error(GQA_DEVERR_SEQLEN);
    len = 0;
  }
  it.len = len;
  it.t_begin = it.split * p.chunk;
  it.t_end = min(len, it.t_begin + p.chunk);
  it.h0 = it.g * p.G + it.hsl * heads_per_cta;
  it.nh = min(heads_per_cta, p.G - it.hsl * heads_per_cta);
  return it;
}

template <typename T>
__device__ __forceinline__ void store_out(T* dst, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* dst, float v) {
  *dst = v;
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, float v) {
  *dst = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------------------
// bf16 tensor-core decode

template <int D>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DecodeParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;

  const DecItem w = decode_item(p, kDecHeadsPerCta);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);

  if (w.t_begin >= w.t_end) {
    // No key of this sequence falls in this split. With a single split this
    // CTA owns the output (len_b == 0 -> zeros); otherwise the combine only
    // reads the first ceil(len_b / chunk) splits.
    if (p.nsplit == 1)
      for (int i = threadIdx.x; i < w.nh * D; i += blockDim.x)
        out[((size_t)w.b * p.H + w.h0 + i / D) * D + (i % D)] = __float2bfloat16_rn(0.f);
    return;
  }
  const int ntiles = (w.t_end - w.t_begin + kDecTileKeys - 1) / kDecTileKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      const uint64_t policy = l2_policy_evict_first();
      const int row_base = w.unit * p.S_max;
      int issued = 0;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % C::kStages;
        if (it >= C::kStages && !mbar_wait_bounded(&empty[s], ((it / C::kStages) - 1) & 1)) break;
        const int t0 = w.t_begin + it * kDecTileKeys;
        const int rows = min(kDecTileKeys, w.t_end - t0);
        const int nbox = (rows + kDecBoxRows - 1) / kDecBoxRows;
        uint8_t* ks = smem + s * C::kStageBytes;
        uint8_t* vs = ks + C::kTileBytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * kDecBoxRows * 128 * C::kHalves * 2));
        for (int bx = 0; bx < nbox; ++bx) {
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf) {
            const int off = hf * C::kHalfBytes + bx * kDecBoxRows * 128;
            tma_load_2d(ks + off, &tm_k, hf * 64, row_base + t0 + bx * kDecBoxRows, &full[s], policy);
            tma_load_2d(vs + off, &tm_v, hf * 64, row_base + t0 + bx * kDecBoxRows, &full[s], policy);
          }
        }
        ++issued;
      }
      // Wait for this CTA's own loads to land before the block may exit.
      for (int it = max(0, issued - C::kStages); it < issued; ++it)
        mbar_wait_bounded(&full[it % C::kStages], (it / C::kStages) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Q^T as the B operand (k = dims, n = heads): lane holds head lane/4,
  // dims 2*(lane%4) + {0,1} (b0) and + 8 (b1) of every 16-dim step.
  uint32_t qf[D / 16][2];
  {
    const int hn = lane >> 2;
    const bool hv = hn < w.nh;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) +
                                                             ((size_t)w.b * p.H + w.h0 + (hv ? hn : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t lo = __ldg(qrow + ks * 8 + (lane & 3));
      const uint32_t hi = __ldg(qrow + ks * 8 + 4 + (lane & 3));
      qf[ks][0] = hv ? lo : 0u;
      qf[ks][1] = hv ? hi : 0u;
    }
  }

  // Running state for heads a = 2*(lane%4) and b = a + 1 (log2 units).
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  float o[D / 16][4];
#pragma unroll
  for (int md = 0; md < D / 16; ++md) o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;

  const int kb = warp * 16;  // this warp's 16 keys inside every tile
  // ldmatrix row/column assignment (lane -> 8x8 matrix lane/8)
  const int k_row = kb + (lane & 7) + ((lane >> 3) & 1) * 8;  // K: matrices (r0-7,c0-7) (r8-15,c0-7) (r0-7,c8-15) ...
  const int k_col8 = (lane >> 4);
  const int v_row = kb + (lane & 7) + (lane >> 4) * 8;  // V^T: matrices (d0-7,k0-7) (d8-15,k0-7) (d0-7,k8-15) ...
  const int v_col8 = (lane >> 3) & 1;

  for (int it = 0; it < ntiles; ++it) {
    const int s = it % C::kStages;
    if (!mbar_wait_bounded(&full[s], (it / C::kStages) & 1)) break;
    const int t0 = w.t_begin + it * kDecTileKeys;
    const int rows = min(kDecTileKeys, w.t_end - t0);
    if (kb < rows) {
      const uint32_t k_base = smem_u32(smem + s * C::kStageBytes);
      const uint32_t v_base = k_base + C::kTileBytes;

      // S^T = K * Q^T
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int chunk = ks * 2 + k_col8;  // 16-byte chunk index along the row
        const uint32_t addr = k_base + (chunk >> 3) * C::kHalfBytes + sw128(k_row, chunk & 7);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(addr, a0, a1, a2, a3);
        mma_bf16_16816(c, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
      }

      // online softmax over this block's keys (key kb + lane/4 in c0/c1, +8 in c2/c3)
      const int key0 = kb + (lane >> 2);
      const bool v0 = key0 < rows, v1 = key0 + 8 < rows;
      const float x0 = v0 ? c[0] * p.scale_log2 : -INFINITY;
      const float x1 = v0 ? c[1] * p.scale_log2 : -INFINITY;
      const float x2 = v1 ? c[2] * p.scale_log2 : -INFINITY;
      const float x3 = v1 ? c[3] * p.scale_log2 : -INFINITY;
      float mx_a = fmaxf(x0, x2), mx_b = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
      }
      const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
      const float al_a = fast_exp2(m_a - mn_a), al_b = fast_exp2(m_b - mn_b);
      m_a = mn_a;
      m_b = mn_b;
      const float p0 = fast_exp2(x0 - mn_a), p1 = fast_exp2(x1 - mn_b);
      const float p2 = fast_exp2(x2 - mn_a), p3 = fast_exp2(x3 - mn_b);
      l_a = l_a * al_a + p0 + p2;
      l_b = l_b * al_b + p1 + p3;
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        o[md][0] *= al_a;
        o[md][1] *= al_b;
        o[md][2] *= al_a;
        o[md][3] *= al_b;
      }

      // P^T (k = keys, n = heads) from the S^T accumulator layout
      const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
      const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));

      // keys of this block past the end of the sequence: zero their V^T
      // entries (the rows may hold anything, NaN included)
      uint32_t mask_lo = 0xffffffffu, mask_hi = 0xffffffffu;
      if (kb + 16 > rows) {
        const int lim = rows - kb;
        const int kk = 2 * (lane & 3);
        mask_lo = (kk < lim ? 0x0000ffffu : 0u) | (kk + 1 < lim ? 0xffff0000u : 0u);
        mask_hi = (kk + 8 < lim ? 0x0000ffffu : 0u) | (kk + 9 < lim ? 0xffff0000u : 0u);
      }

      // O^T += V^T * P^T
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        const int chunk = md * 2 + v_col8;
        const uint32_t addr = v_base + (chunk >> 3) * C::kHalfBytes + sw128(v_row, chunk & 7);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(addr, a0, a1, a2, a3);
        mma_bf16_16816(o[md], a0 & mask_lo, a1 & mask_lo, a2 & mask_hi, a3 & mask_hi, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------------------------------------------------------- merge
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
  }
  float* red_m = reinterpret_cast<float*>(smem);                  // [4][8]
  float* red_l = red_m + kDecConsumerWarps * kDecHeadsPerCta;     // [4][8]
  float* red_o = red_l + kDecConsumerWarps * kDecHeadsPerCta;     // [4][8][D]
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");  // stage buffers now free
  {
    const int ha = 2 * (lane & 3);
    if (lane < 4) {
      red_m[warp * 8 + ha] = m_a;
      red_m[warp * 8 + ha + 1] = m_b;
      red_l[warp * 8 + ha] = l_a;
      red_l[warp * 8 + ha + 1] = l_b;
    }
    float* ow = red_o + warp * kDecHeadsPerCta * D;
    const int dr = lane >> 2;
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      ow[ha * D + md * 16 + dr] = o[md][0];
      ow[(ha + 1) * D + md * 16 + dr] = o[md][1];
      ow[ha * D + md * 16 + dr + 8] = o[md][2];
      ow[(ha + 1) * D + md * 16 + dr + 8] = o[md][3];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");

  const size_t part = ((size_t)w.unit * p.nsplit + w.split) * p.G + (size_t)w.hsl * kDecHeadsPerCta;
  for (int i = threadIdx.x; i < w.nh * D; i += kDecConsumerWarps * 32) {
    const int h = i / D, dim = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kDecConsumerWarps; ++ww) M = fmaxf(M, red_m[ww * 8 + h]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int ww = 0; ww < kDecConsumerWarps; ++ww) {
      const float f = fast_exp2(red_m[ww * 8 + h] - M);
      L += red_l[ww * 8 + h] * f;
      O += red_o[(ww * kDecHeadsPerCta + h) * D + dim] * f;
    }
    if (p.nsplit == 1) {
      out[((size_t)w.b * p.H + w.h0 + h) * D + dim] = __float2bfloat16_rn(O / L);
    } else {
      p.ws_o[(part + h) * D + dim] = O;
      if (dim == 0) p.ws_ml[part + h] = make_float2(M, L);
    }
  }
}

// ---------------------------------------------------------------------------
// float32 decode (plain FMA): one warp per query head, lanes over keys for
// the scores and over dims for the weighted sum of V.

constexpr int kDecF32Threads = 128;
constexpr int kDecF32Keys = 32;
constexpr int kDecF32HeadsPerWarp = 4;
constexpr int kDecF32HeadsPerCta = kDecF32HeadsPerWarp * (kDecF32Threads / 32);

template <int D>
__global__ void __launch_bounds__(kDecF32Threads) decode_f32_kernel(const float* __restrict__ k_cache,
                                                                    const float* __restrict__ v_cache,
                                                                    const DecodeParams p) {
  __shared__ float qs[kDecF32HeadsPerCta][D];
  __shared__ float ks[kDecF32Keys][D + 1];
  __shared__ float vs[kDecF32Keys][D];
  const DecItem w = decode_item(p, kDecF32HeadsPerCta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* out = static_cast<float*>(p.out);
  if (w.t_begin >= w.t_end) {
    if (p.nsplit == 1)
      for (int i = threadIdx.x; i < w.nh * D; i += blockDim.x)
        out[((size_t)w.b * p.H + w.h0 + i / D) * D + (i % D)] = 0.f;
    return;
  }
  const float* q = static_cast<const float*>(p.q);
  for (int i = threadIdx.x; i < w.nh * D; i += blockDim.x)
    qs[i / D][i % D] = q[((size_t)w.b * p.H + w.h0 + i / D) * D + (i % D)];

  float m[kDecF32HeadsPerWarp], l[kDecF32HeadsPerWarp], o[kDecF32HeadsPerWarp][D / 32];
#pragma unroll
  for (int j = 0; j < kDecF32HeadsPerWarp; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[j][c] = 0.f;
  }
  const size_t row0 = (size_t)w.unit * p.S_max;
  for (int t0 = w.t_begin; t0 < w.t_end; t0 += kDecF32Keys) {
    const int rows = min(kDecF32Keys, w.t_end - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < kDecF32Keys * D; i += blockDim.x) {
      const int r = i / D, c = i % D;
      const bool ok = r < rows;
      ks[r][c] = ok ? k_cache[(row0 + t0 + r) * D + c] : 0.f;
      vs[r][c] = ok ? v_cache[(row0 + t0 + r) * D + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kDecF32HeadsPerWarp; ++j) {
      const int h = warp * kDecF32HeadsPerWarp + j;
      if (h >= w.nh) break;
      float sc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) sc = fmaf(qs[h][c], ks[lane][c], sc);
      const float x = lane < rows ? sc * p.scale_log2 : -INFINITY;
      float mx = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[j], mx);
      const float al = exp2f(m[j] - mn);
      const float pr = exp2f(x - mn);
      float ps = pr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[j] = l[j] * al + ps;
      m[j] = mn;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) o[j][c] *= al;
      for (int t = 0; t < rows; ++t) {
        const float pt = __shfl_sync(0xffffffffu, pr, t);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) o[j][c] = fmaf(pt, vs[t][lane + 32 * c], o[j][c]);
      }
    }
  }
  const size_t part = ((size_t)w.unit * p.nsplit + w.split) * p.G + (size_t)w.hsl * kDecF32HeadsPerCta;
#pragma unroll
  for (int j = 0; j < kDecF32HeadsPerWarp; ++j) {
    const int h = warp * kDecF32HeadsPerWarp + j;
    if (h >= w.nh) break;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const int dim = lane + 32 * c;
      if (p.nsplit == 1) {
        out[((size_t)w.b * p.H + w.h0 + h) * D + dim] = o[j][c] / l[j];
      } else {
        p.ws_o[(part + h) * D + dim] = o[j][c];
        if (dim == 0) p.ws_ml[part + h] = make_float2(m[j], l[j]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Split-KV combine: out[b,h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,
// M = max_s m_s, over the ceil(len_b / chunk) splits that hold keys.
// One CTA of D threads per (b, h).

template <typename OutT>
__global__ void decode_combine_kernel(OutT* __restrict__ out, const float* __restrict__ ws_o,
                                      const float2* __restrict__ ws_ml, const int32_t* __restrict__ seqlens, int H,
                                      int K, int S_max, int G, int chunk, int nsplit, int D) {
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int g = h / G, j = h % G;
  int len = __ldg(seqlens + b);
  if (len < 0 || len > S_max) len = 0;
  const int ns = (len + chunk - 1) / chunk;
  const size_t base = ((size_t)(b * K + g) * nsplit) * G + j;  // split s at base + s*G
  const int dim = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldg(&ws_ml[base + (size_t)s * G].x));
  float L = 0.f, acc = 0.f;
  int s = 0;
  for (; s + 4 <= ns; s += 4) {
    float2 ml[4];
    float ov[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ml[u] = __ldg(&ws_ml[base + (size_t)(s + u) * G]);
      ov[u] = __ldg(&ws_o[(base + (size_t)(s + u) * G) * D + dim]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float f = fast_exp2(ml[u].x - M);
      L += ml[u].y * f;
      acc += ov[u] * f;
    }
  }
  for (; s < ns; ++s) {
    const float2 ml = __ldg(&ws_ml[base + (size_t)s * G]);
    const float f = fast_exp2(ml.x - M);
    L += ml.y * f;
    acc += __ldg(&ws_o[(base + (size_t)s * G) * D + dim]) * f;
  }
  store_out<OutT>(out + (size_t)bh * D + dim, ns > 0 ? acc / L : 0.f);
}

}  // namespace gqa
