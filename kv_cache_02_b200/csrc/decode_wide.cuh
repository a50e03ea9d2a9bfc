// GQA decode for wide groups (64 query heads per KV head, e.g. multi-query
// attention) on the 5th-generation tensor cores.
//
// With G = 64 every cached key feeds 64 heads: 64 flop per byte, too much for
// warp-level MMAs fed from shared memory. Here one CTA (one per SM) serves the
// 64 heads of a group from every K/V tile it loads:
//   S[64 heads x 128 keys] = Q[64 x d] K^T[d x 128]    tcgen05.mma M=64, fp32 in TMEM
//   softmax over keys: an M=64 accumulator puts row r in TMEM lane
//       (r mod 16) + 32 * (r / 16), so lanes 0..15 of the four softmax warps
//       each own one head's whole row: max, exp2 and sum stay in the thread
//   P (bf16) into shared memory as the K-major operand
//   O[64 x d] += P[64 x 128 keys] V[128 keys x d]      tcgen05.mma, V MN-major
// The accumulator is rescaled (conditionally, when a head's maximum grows by
// more than 2^8) with tcgen05.ld/st by its owner. Work items (b, g, split,
// slice of 64 heads) come from the same tagged counter as the narrow-group
// kernel; partials are merged by decode_combine_kernel.
//
// Warp roles: 0-3 softmax and epilogue, 4 TMA producer, 5 TMEM allocation
// and the single MMA-issuing thread.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "tcgen05.cuh"

namespace gqa {

constexpr int kWideHeads = 64;    // query heads per CTA: the MMA N of both products
constexpr int kWideKeys = 128;    // keys per tile: the M of S^T and the K of O^T
constexpr int kWideThreads = 192;
constexpr int kWideTmemCols = 512;
constexpr int kWideBox = 64;      // TMA box height of full tiles (the tail uses kDecBoxRows)

struct WideCfg {  // head dim 128
  static constexpr int D = 128;
  static constexpr int kStages = 3;
  static constexpr int kHalf = kWideKeys * 128;        // one 64-dim half of a K or V tile: 16 KB
  static constexpr int kTile = 2 * kHalf;              // K (or V) tile: 32 KB
  static constexpr int kStage = 2 * kTile;             // K then V
  static constexpr int kQHalf = kWideHeads * 128;      // 8 KB
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQOff + 2 * kQHalf;
  static constexpr int kPOff = kKVOff + kStages * kStage;
  static constexpr int kPHalf = kWideHeads * 128;         // P: 64 heads x 64 keys, 8 KB
  static constexpr int kPBytes = 2 * kPHalf;               // 128 keys
  static constexpr int kInfoOff = kPOff + kPBytes;
  static constexpr int kBarOff = kInfoOff + kStages * 16;
  static constexpr int kNumBars = 2 + 2 * kStages + 4 + 4;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kSCol = 0;    // two S buffers: columns [0, 128) and [128, 256)
  static constexpr int kOCol = 256;  // O: columns [256, 384)
};

// TMA loads of `rows` keys of one unit: 64-row boxes, then 16-row boxes for the tail
__device__ __forceinline__ void wide_issue_tile(uint8_t* stage, uint64_t* full, const CUtensorMap* tm_k64,
                                                const CUtensorMap* tm_v64, const CUtensorMap* tm_k16,
                                                const CUtensorMap* tm_v16, int row0, int rows, uint64_t policy) {
  using C = WideCfg;
  const int n64 = rows / kWideBox;
  const int rem = rows - n64 * kWideBox;
  const int n16 = (rem + kDecBoxRows - 1) / kDecBoxRows;
  mbar_arrive_expect_tx(full, (uint32_t)((n64 * kWideBox + n16 * kDecBoxRows) * 128 * 2 * 2));
  for (int bx = 0; bx < n64; ++bx)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int off = hf * C::kHalf + bx * kWideBox * 128;
      tma_load_2d(stage + off, tm_k64, hf * 64, row0 + bx * kWideBox, full, policy);
      tma_load_2d(stage + C::kTile + off, tm_v64, hf * 64, row0 + bx * kWideBox, full, policy);
    }
  for (int bx = 0; bx < n16; ++bx)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = n64 * kWideBox + bx * kDecBoxRows;
      const int off = hf * C::kHalf + r * 128;
      tma_load_2d(stage + off, tm_k16, hf * 64, row0 + r, full, policy);
      tma_load_2d(stage + C::kTile + off, tm_v16, hf * 64, row0 + r, full, policy);
    }
}

__global__ void __launch_bounds__(kWideThreads, 1)
    decode_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k64,
                       const __grid_constant__ CUtensorMap tm_v64, const __grid_constant__ CUtensorMap tm_k16,
                       const __grid_constant__ CUtensorMap tm_v16, const DecodeParams p) {
  using C = WideCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem[];
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + C::kInfoOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + C::kStages;
  uint64_t* s_full = kv_empty + C::kStages;  // [2]
  uint64_t* s_free = s_full + 2;             // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* o_free = pv_done + 1;
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(o_free, 128);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, kWideTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k64);
      prefetch_tensormap(&tm_v64);
      const uint64_t policy = l2_policy_evict_first();
      const uint64_t q_policy = l2_policy_evict_last();
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      int it = 0, nq = 0;
      bool ok = true;
      for (int k = 0;; ++k) {
        // the first item of each CTA is its block index; later ones come from the counter
        const int item = k == 0 ? (int)blockIdx.x : (int)gridDim.x + take_ticket(p.ws_queue, p.tag) - 1;
        if (item < 0 || item >= p.nitems) break;
        const ItemCoord c = item_coord_n(p, item, kWideHeads);
        const int raw = __ldg(p.seqlens + c.b);
        const int len = valid_len(raw + p.len_add, p.S_max);
        if (c.g == 0 && c.split == 0 && c.hsl == 0 && !p.len_add && len != raw) raise_error(GQA_DEVERR_SEQLEN);
        const int t_begin = c.split * p.chunk;
        const int t_end = min(len, t_begin + p.chunk);
        if (t_begin >= t_end) {
          if (c.split == 0) {
            uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)c.b * p.H + c.h0) * D);
            for (int i = 0; i < c.nh * D / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
          }
          continue;
        }
        // Q of this item's 64 heads
        if (nq >= 1 && !(ok = mbar_wait_bounded(q_empty, (nq - 1) & 1))) break;
        mbar_arrive_expect_tx(q_full, 2 * C::kQHalf);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d(smem + C::kQOff + hf * C::kQHalf, &tm_q, hf * 64, c.b * p.H + c.h0, q_full, q_policy);
        ++nq;
        const int ntiles = (t_end - t_begin + kWideKeys - 1) / kWideKeys;
        const int row_base = c.unit * p.S_max;
        for (int tt = 0; tt < ntiles && ok; ++tt, ++it) {
          const int s = it % C::kStages;
          if (it >= C::kStages) ok = mbar_wait_bounded(&kv_empty[s], ((it / C::kStages) - 1) & 1);
          if (!ok) break;
          const int t0 = t_begin + tt * kWideKeys;
          const int rows = min(kWideKeys, t_end - t0);
          info[s] = StageInfo{item, rows, (tt == 0 ? 1 : 0) | (tt == ntiles - 1 ? 2 : 0), -1};
          wide_issue_tile(smem + C::kKVOff + s * C::kStage, &kv_full[s], &tm_k64, &tm_v64, &tm_k16, &tm_v16,
                          row_base + t0, rows, policy);
        }
        if (!ok) break;
      }
      if (ok) {
        const int s = it % C::kStages;
        if (it >= C::kStages) ok = mbar_wait_bounded(&kv_empty[s], ((it / C::kStages) - 1) & 1);
        if (ok) {
          info[s] = StageInfo{-1, 0, 0, -1};
          mbar_arrive(&kv_full[s]);
          ++it;
        }
      }
      for (int j = max(0, it - C::kStages); j < it; ++j) mbar_wait_bounded(&kv_full[j % C::kStages], (j / C::kStages) & 1);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kWideHeads, kWideKeys, false, false);  // Q K^T
      constexpr uint32_t idesc_o = idesc_bf16_f32(kWideHeads, D, false, true);          // P V, V MN-major
      const uint32_t q_addr = smem_u32(smem + C::kQOff);
      const uint32_t p_addr = smem_u32(smem + C::kPOff);
      int nitem = 0;  // items started
      int prev_first = 0, prev_ord = 0;  // tile j-1: opened its item; ordinal of its item
      int cur_ord = 0;
      bool ok = true;
      int j = 0;
      auto issue_pv = [&](int t, int first, int ord) -> bool {
        if (!mbar_wait_bounded(p_full, t & 1)) return false;
        // the first PV of an item overwrites O^T: the previous item's epilogue must have read it
        if (first && ord >= 1 && !mbar_wait_bounded(o_free, (ord - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + C::kKVOff + (t % C::kStages) * C::kStage + C::kTile);
#pragma unroll
        for (int kk = 0; kk < kWideKeys / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(p_addr + (kk >> 2) * C::kPHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, C::kHalf, 1024);
          tc_mma(tmem + C::kOCol, ad, bd, idesc_o, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(pv_done);
        tc_commit(&kv_empty[t % C::kStages]);
        return true;
      };
      for (;; ++j) {
        const int s = j % C::kStages;
        if (!(ok = mbar_wait_bounded(&kv_full[s], (j / C::kStages) & 1))) break;
        const StageInfo si = info[s];
        if (si.item < 0) break;
        if (si.flags & 1) {
          if (!(ok = mbar_wait_bounded(q_full, nitem & 1))) break;
          cur_ord = nitem++;
        }
        if (j >= 2 && !(ok = mbar_wait_bounded(&s_free[j & 1], ((j >> 1) - 1) & 1))) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + C::kKVOff + s * C::kStage);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(q_addr + (kk >> 2) * C::kQHalf + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + (kk >> 2) * C::kHalf + off, 16, 1024);
          tc_mma(tmem + C::kSCol + (uint32_t)((j & 1) * kWideKeys), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[j & 1]);
        if (si.flags & 2) tc_commit(q_empty);  // the item's last S: Q may be replaced
        if (j >= 1 && !(ok = issue_pv(j - 1, prev_first, prev_ord))) break;
        prev_first = si.flags & 1;
        prev_ord = cur_ord;
      }
      if (ok && j >= 1) issue_pv(j - 1, prev_first, prev_ord);
      tc_commit(mma_done);  // completes when every MMA issued above has finished
      mbar_wait_bounded(mma_done, 0);
    }
  } else {
    // ---------------------------------------------------- softmax / epilogue
    // lanes 0..15 of warp w own head r = 16 w + lane (TMEM lane 32 w + lane);
    // lanes 16..31 run the same instructions on rows that hold no head
    const int t = threadIdx.x;
    const int r = warp * 16 + (lane & 15);
    const bool owner = lane < 16;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* prow = smem + C::kPOff + r * 128;
    float m_used = -INFINITY, l = 0.f;
    ItemCoord c{};
    for (int j = 0;; ++j) {
      const int s = j % C::kStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&kv_full[s], (j / C::kStages) & 1))) break;
      const StageInfo si = info[s];
      if (si.item < 0) break;
      const bool first = si.flags & 1;
      if (first) {
        c = item_coord_n(p, si.item, kWideHeads);
        m_used = -INFINITY;
        l = 0.f;
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      float x[2 * 64];
      {
        float a[64], bb[64];
        tmem_ld64(lane_addr + C::kSCol + (uint32_t)((j & 1) * kWideKeys), a);
        tmem_ld64(lane_addr + C::kSCol + (uint32_t)((j & 1) * kWideKeys + 64), bb);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          x[i] = a[i];
          x[64 + i] = bb[i];
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[j & 1]);

      float mt = -INFINITY;
#pragma unroll
      for (int k = 0; k < kWideKeys; ++k) {
        x[k] = k < si.rows ? x[k] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, x[k]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_used + 8.f) {  // first tile of an item: m_used = -inf
        const float mn = fmaxf(mt, m_used);
        alpha = fast_exp2(m_used - mn);
        rescale = !first;
        m_used = mn;
      }
      float sum = 0.f;
      uint32_t pk[kWideKeys / 2];
#pragma unroll
      for (int k = 0; k < kWideKeys; k += 2) {
        const float p0 = fast_exp2(x[k] - m_used);
        const float p1 = fast_exp2(x[k + 1] - m_used);
        sum += p0 + p1;
        pk[k / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + sum;
      // the P buffer and O are free once the previous tile's PV has finished
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (j - 1) & 1))) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale && owner)) {  // lanes that keep their max scale by 1
        const float a = (rescale && owner) ? alpha : 1.f;
        float o[32];
#pragma unroll 1
        for (int cb = 0; cb < D; cb += 32) {
          tmem_ld32(lane_addr + C::kOCol + cb, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= a;
          tmem_st32(lane_addr + C::kOCol + cb, o);
        }
        tc_wait_st();
      }
      if (t >= si.rows) {  // key rows past the sequence: zero V (0 * NaN would poison the sum)
        uint8_t* vrow = smem + C::kKVOff + s * C::kStage + C::kTile + t * 128;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(vrow + hf * C::kHalf + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      if (owner) {
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
          const uint32_t off = (uint32_t)((ch >> 3) * C::kPHalf) + ((((uint32_t)(ch & 7)) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(prow + off) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(p_full);

      if (si.flags & 2) {
        // ---- item epilogue: O / l -> out (one split) or the split's partial
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, j & 1))) break;
        tc_fence_after();
        float o[D];
        tmem_ld64(lane_addr + C::kOCol, *reinterpret_cast<float(*)[64]>(o));
        tmem_ld64(lane_addr + C::kOCol + 64, *reinterpret_cast<float(*)[64]>(o + 64));
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(o_free);
        const int len = valid_len(__ldg(p.seqlens + c.b) + p.len_add, p.S_max);
        const int ns = (len + p.chunk - 1) / p.chunk;
        if (owner && ns == 1) {
          const float inv = 1.f / l;
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                ((size_t)c.b * p.H + c.h0 + r) * D);
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            dst[i] = make_uint4(pack_bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv),
                                pack_bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                pack_bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                pack_bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
        } else if (owner) {
          const size_t part = ((size_t)c.unit * p.nsplit + c.split) * p.G + (size_t)c.hsl * kWideHeads + r;
          float4* dst = reinterpret_cast<float4*>(p.ws_o + part * D);
#pragma unroll
          for (int i = 0; i < D / 4; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          p.ws_ml[part] = make_float2(m_used, l);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kWideTmemCols);
  }
}

}  // namespace gqa
