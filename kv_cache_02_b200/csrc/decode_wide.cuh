// GQA decode for wide groups (64 query heads per KV head, e.g. multi-query
// attention) on the 5th-generation tensor cores.
//
// With G = 64 every cached key feeds 64 heads: 64 flop per byte, too much for
// warp-level MMAs fed from shared memory. Here one CTA (one per SM) serves the
// 64 heads of a group from every K/V tile it loads:
//   S[64 heads x 128 keys] = Q[64 x d] K^T[d x 128]    tcgen05.mma M=64, fp32 in TMEM
//   softmax over keys: an M=64 accumulator puts row r in TMEM lane
//       (r mod 16) + 32 * (r / 16); the 16-lane TMEM load shape spreads the
//       16 rows of a softmax warp over all its 32 threads, a quad of threads
//       per pair of heads, each thread 32 keys of both
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
// Keys of the first work item warmed in L2 before the grid dependency: with
// one item per SM this is the first two tiles (back to back MQA calls 6 % faster
// than without it, 0 % to 2 % slower in isolation, measured; the whole item was slower).
#ifndef GQA_WIDE_WARM_KEYS
#define GQA_WIDE_WARM_KEYS 256
#endif
constexpr int kWideWarmKeys = GQA_WIDE_WARM_KEYS;

#ifndef GQA_WIDE_STAGES
#define GQA_WIDE_STAGES 3
#endif

struct WideCfg {  // head dim 128
  static constexpr int D = 128;
  static constexpr int kStages = GQA_WIDE_STAGES;
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

// The contiguous cache: the tile's rows start at row0.
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

// The producer warp of the paged kernel. Lane 0 takes the work items, waits
// for free stages and loads Q; the 32 lanes hold a window of 32 entries of
// the item's block-table row (lane j: block win + j, loaded in one coalesced
// load at the item's start and again when a tile passes the window), and
// each TMA box of a tile is issued by its own lane, which finds its block
// with one shuffle. A box lies inside one block: 64-row boxes when the block
// size is a multiple of 64, 16-row boxes otherwise and for a tile's tail
// (block sizes are multiples of 16). Against one thread issuing every box
// and reading the table a tile ahead, MQA over a 128K-token context at block
// size 16 (eight 16-row boxes per 128-key tile, 32 TMA instructions) went
// from 0.31 to 0.46 of the copy bandwidth (the contiguous cache: 0.54).
__device__ __forceinline__ void wide_produce_paged(const DecodeParams& p, uint8_t* smem, StageInfo* info,
                                                   uint64_t* kv_full, uint64_t* kv_empty, uint64_t* q_full,
                                                   uint64_t* q_empty, const CUtensorMap* tm_q,
                                                   const CUtensorMap* tm_k64, const CUtensorMap* tm_v64,
                                                   const CUtensorMap* tm_k16, const CUtensorMap* tm_v16, int lane) {
  using C = WideCfg;
  constexpr int D = C::D;
  constexpr unsigned kAll = 0xffffffffu;
  if (lane == 0) {
    prefetch_tensormap(tm_k16);
    prefetch_tensormap(tm_v16);
  }
  const uint64_t policy = l2_policy_evict_first();
  const uint64_t q_policy = l2_policy_evict_last();
  const int bs = p.block_size;
  const bool big = bs % kWideBox == 0;  // a 64-key group lies inside one block
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  int it = 0, nq = 0;
  bool ok = true;
  for (int k = 0;; ++k) {
    // the first item of each CTA is its block index; later ones come from the counter
    int ticket = 1;
    if (k > 0) {
      if (lane == 0) ticket = take_ticket(p.ws_queue, p.tag);
      ticket = __shfl_sync(kAll, ticket, 0);
    }
    const int item = k == 0 ? (int)blockIdx.x : (int)gridDim.x + ticket - 1;
    if (ticket <= 0 || item >= p.nitems) break;
    const ItemCoord c = item_coord_n(p, item, kWideHeads);
    const int raw = __ldg(p.seqlens + c.b);
    const int len = valid_len(raw + p.len_add, p.S_max);
    if (lane == 0 && c.g == 0 && c.split == 0 && c.hsl == 0 && !p.len_add && len != raw)
      raise_error(GQA_DEVERR_SEQLEN);
    const int t_begin = c.split * p.chunk;
    const int t_end = min(len, t_begin + p.chunk);
    if (t_begin >= t_end) {
      if (c.split == 0) {  // an empty sequence: zeros for this item's heads
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)c.b * p.H + c.h0) * D);
        for (int i = lane; i < c.nh * D / 8; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      continue;
    }
    // Q of this item's 64 heads
    if (lane == 0) {
      if (nq >= 1) ok = mbar_wait_bounded(q_empty, (nq - 1) & 1);
      if (ok) {
        mbar_arrive_expect_tx(q_full, 2 * C::kQHalf);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d(smem + C::kQOff + hf * C::kQHalf, tm_q, hf * 64, c.b * p.H + c.h0, q_full, q_policy);
      }
    }
    ok = __shfl_sync(kAll, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    ++nq;
    const int ntiles = (t_end - t_begin + kWideKeys - 1) / kWideKeys;
    const int32_t* trow = p.block_table + (size_t)c.b * p.max_blocks;
    const int blk_end = (t_end - 1) / bs + 1;  // the item's blocks: [t_begin / bs, blk_end)
    int win = t_begin / bs;                    // lane j holds the entry of block win + j
    int ent = win + lane < blk_end ? __ldg(trow + win + lane) : 0;
    for (int tt = 0; tt < ntiles && ok; ++tt, ++it) {
      const int s = it % C::kStages;
      const int t0 = t_begin + tt * kWideKeys;
      const int rows = min(kWideKeys, t_end - t0);
      const int last_blk = (t0 + rows - 1) / bs;
      if (last_blk >= win + 32) {  // the tile's blocks are past the window: the next 32
        win = t0 / bs;
        ent = win + lane < blk_end ? __ldg(trow + win + lane) : 0;
      }
      if (lane == 0 && it >= C::kStages) ok = mbar_wait_bounded(&kv_empty[s], ((it / C::kStages) - 1) & 1);
      ok = __shfl_sync(kAll, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      // boxes: n64 of 64 rows, then n16 of 16 rows; box i is issued by lane i
      const int n64 = big ? rows / kWideBox : 0;
      const int n16 = (rows - n64 * kWideBox + kDecBoxRows - 1) / kDecBoxRows;
      const int nbox = n64 + n16;
      const int bi = lane < nbox ? lane : 0;
      const int r0 = bi < n64 ? bi * kWideBox : n64 * kWideBox + (bi - n64) * kDecBoxRows;  // the box's first key
      const int e = __shfl_sync(kAll, ent, (t0 + r0) / bs - win);
      uint8_t* stage = smem + C::kKVOff + s * C::kStage;
      if (lane == 0) {
        info[s] = StageInfo{item, rows,
                            (tt == 0 ? kTileFirst : 0) | (tt == ntiles - 1 ? kTileLast : 0) |
                                (len <= p.chunk ? kUnitSingleSplit : 0),
                            -1};
        mbar_arrive_expect_tx(&kv_full[s], (uint32_t)((n64 * kWideBox + n16 * kDecBoxRows) * 128 * 2 * 2));
      }
      __syncwarp();
      if (lane < nbox) {
        const int brow = paged_row(p, e, c.g, t0 + r0);
        const bool b64 = bi < n64;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int off = hf * C::kHalf + r0 * 128;
          tma_load_2d(stage + off, b64 ? tm_k64 : tm_k16, hf * 64, brow, &kv_full[s], policy);
          tma_load_2d(stage + C::kTile + off, b64 ? tm_v64 : tm_v16, hf * 64, brow, &kv_full[s], policy);
        }
      }
    }
    if (!ok) break;
  }
  if (lane == 0) {
    leave_queue(p.ws_queue, p.tag);
    // no more work: a record without loads ends the consumers' loop
    if (ok) {
      const int s = it % C::kStages;
      if (it >= C::kStages) ok = mbar_wait_bounded(&kv_empty[s], ((it / C::kStages) - 1) & 1);
      if (ok) {
        info[s] = StageInfo{-1, 0, 0, -1};
        mbar_arrive(&kv_full[s]);
        ++it;
      }
    }
    // this CTA's own loads must land before the block may exit
    for (int j = max(0, it - C::kStages); j < it; ++j)
      mbar_wait_bounded(&kv_full[j % C::kStages], (j / C::kStages) & 1);
  }
}

// One tile of the online softmax for the two heads a thread holds. x: the raw
// scores of 32 keys of head a (x[4i], x[4i+1]) and of head b (x[4i+2],
// x[4i+3]), key 8i + 2 qi + {0, 1}. Keys at or past `rows` do not count. The
// running maxima m_a, m_b are in log2 units with the scale applied and are
// common to the quad; l_a, l_b are this thread's share of the sums. alpha_a,
// alpha_b: the factors O must be multiplied by (1 when the maximum is kept).
// With a positive scale the maximum is taken over the raw scores and the
// scale folds into the exponent's multiply-add.
template <bool kPosScale>
__device__ __forceinline__ void wide_softmax_tile(float (&x)[64], int rows, int qi, float sl2, float& m_a,
                                                  float& m_b, float& l_a, float& l_b, uint32_t (&pa)[16],
                                                  uint32_t (&pb)[16], float& alpha_a, float& alpha_b) {
  if constexpr (!kPosScale) {
#pragma unroll
    for (int e = 0; e < 64; ++e) x[e] *= sl2;
  }
  if (rows < kWideKeys) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (8 * i + 2 * qi + (k & 1) >= rows) x[4 * i + k] = -INFINITY;
  }
  float a0 = x[0], a1 = x[1], b0 = x[2], b1 = x[3];
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    a0 = fmaxf(a0, x[4 * i]);
    a1 = fmaxf(a1, x[4 * i + 1]);
    b0 = fmaxf(b0, x[4 * i + 2]);
    b1 = fmaxf(b1, x[4 * i + 3]);
  }
  float ma = fmaxf(a0, a1), mb = fmaxf(b0, b1);
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, off));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
  }
  if constexpr (kPosScale) {
    ma *= sl2;
    mb *= sl2;
  }
  alpha_a = 1.f;
  alpha_b = 1.f;
  if (ma > m_a + 8.f) {  // first tile of an item: m = -inf
    const float mn = fmaxf(ma, m_a);
    alpha_a = fast_exp2(m_a - mn);
    m_a = mn;
  }
  if (mb > m_b + 8.f) {
    const float mn = fmaxf(mb, m_b);
    alpha_b = fast_exp2(m_b - mn);
    m_b = mn;
  }
  const float nma = -m_a, nmb = -m_b;
  float sa = 0.f, sb = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float p0, p1, p2, p3;
    if constexpr (kPosScale) {
      p0 = fast_exp2(fmaf(x[4 * i], sl2, nma));
      p1 = fast_exp2(fmaf(x[4 * i + 1], sl2, nma));
      p2 = fast_exp2(fmaf(x[4 * i + 2], sl2, nmb));
      p3 = fast_exp2(fmaf(x[4 * i + 3], sl2, nmb));
    } else {
      p0 = fast_exp2(x[4 * i] + nma);
      p1 = fast_exp2(x[4 * i + 1] + nma);
      p2 = fast_exp2(x[4 * i + 2] + nmb);
      p3 = fast_exp2(x[4 * i + 3] + nmb);
    }
    sa += p0 + p1;
    sb += p2 + p3;
    pa[i] = pack_bf16x2(p0, p1);
    pb[i] = pack_bf16x2(p2, p3);
  }
  l_a = l_a * alpha_a + sa;
  l_b = l_b * alpha_b + sb;
}

template <bool kPaged>
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
    grid_dep_wait();
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  // Launched as a programmatic dependent (as the narrow-group kernel): until
  // grid_dep_wait() returns only the set-up below, the descriptor prefetch
  // and an L2 warm-up of the first item's key rows (contiguous cache) run,
  // the latter sized by a length that may be stale.
  int spec_first = 0;
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k64);
    prefetch_tensormap(&tm_v64);
    if ((int)blockIdx.x < p.nitems) spec_first = __ldcg(p.seqlens + item_coord_n(p, blockIdx.x, kWideHeads).b);
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
  if (!kPaged && warp == 4 && lane == 0 && (int)blockIdx.x < p.nitems)
    warm_first_item<WideCfg::D * 2>(p, item_coord_n(p, blockIdx.x, kWideHeads), spec_first, kWideWarmKeys);
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if constexpr (kPaged) {
      wide_produce_paged(p, smem, info, kv_full, kv_empty, q_full, q_empty, &tm_q, &tm_k64, &tm_v64, &tm_k16, &tm_v16,
                         lane);
    } else if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      const uint64_t q_policy = l2_policy_evict_last();
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      int it = 0, nq = 0;
      bool ok = true;
      for (int k = 0;; ++k) {
        // the first item of each CTA is its block index; later ones come from the counter
        const int ticket = k == 0 ? 1 : take_ticket(p.ws_queue, p.tag);
        const int item = k == 0 ? (int)blockIdx.x : (int)gridDim.x + ticket - 1;
        if (ticket <= 0 || item >= p.nitems) break;
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
        for (int tt = 0; tt < ntiles && ok; ++tt, ++it) {
          const int s = it % C::kStages;
          const int t0 = t_begin + tt * kWideKeys;
          const int rows = min(kWideKeys, t_end - t0);
          if (it >= C::kStages) ok = mbar_wait_bounded(&kv_empty[s], ((it / C::kStages) - 1) & 1);
          if (!ok) break;
          info[s] = StageInfo{item, rows,
                              (tt == 0 ? kTileFirst : 0) | (tt == ntiles - 1 ? kTileLast : 0) |
                                  (len <= p.chunk ? kUnitSingleSplit : 0),
                              -1};
          wide_issue_tile(smem + C::kKVOff + s * C::kStage, &kv_full[s], &tm_k64, &tm_v64, &tm_k16, &tm_v16,
                          c.unit * p.S_max + t0, rows, policy);
        }
        if (!ok) break;
      }
      leave_queue(p.ws_queue, p.tag);
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
    // The warp runs converged (descriptors are warp-uniform values) and one
    // elected lane issues each tcgen05 instruction: issued from a single-lane
    // branch, each MMA paid for moving its operands to uniform registers.
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_bf16_f32(kWideHeads, kWideKeys, false, false);  // Q K^T
    constexpr uint32_t idesc_o = idesc_bf16_f32(kWideHeads, D, false, true);          // P V, V MN-major
    const uint32_t q_addr = smem_u32(smem + C::kQOff);
    const uint32_t p_addr = smem_u32(smem + C::kPOff);
    int nitem = 0;  // items started
    int prev_first = 0, prev_ord = 0;  // tile j-1: opened its item; ordinal of its item
    int cur_ord = 0;
    bool ok = true;
    int j = 0;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    auto issue_pv = [&](int t, int first, int ord) -> bool {
      if (!wait_all(p_full, t & 1)) return false;
      // the first PV of an item overwrites O^T: the previous item's epilogue must have read it
      if (first && ord >= 1 && !wait_all(o_free, (ord - 1) & 1)) return false;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(smem + C::kKVOff + (t % C::kStages) * C::kStage + C::kTile);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kWideKeys / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(p_addr + (kk >> 2) * C::kPHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, C::kHalf, 1024);
          tc_mma(tmem + C::kOCol, ad, bd, idesc_o, (first && kk == 0) ? 0u : 1u);
        }
      }
      __syncwarp();
      commit(pv_done);
      commit(&kv_empty[t % C::kStages]);
      return true;
    };
    for (;; ++j) {
      const int s = j % C::kStages;
      if (!(ok = wait_all(&kv_full[s], (j / C::kStages) & 1))) break;
      const StageInfo si = info[s];
      if (si.item < 0) break;
      if (si.flags & kTileFirst) {
        if (!(ok = wait_all(q_full, nitem & 1))) break;
        cur_ord = nitem++;
      }
      if (j >= 2 && !(ok = wait_all(&s_free[j & 1], ((j >> 1) - 1) & 1))) break;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(smem + C::kKVOff + s * C::kStage);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(q_addr + (kk >> 2) * C::kQHalf + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + (kk >> 2) * C::kHalf + off, 16, 1024);
          tc_mma(tmem + C::kSCol + (uint32_t)((j & 1) * kWideKeys), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
      commit(&s_full[j & 1]);
      if (si.flags & kTileLast) commit(q_empty);  // the item's last S: Q may be replaced
      if (j >= 1 && !(ok = issue_pv(j - 1, prev_first, prev_ord))) break;
      prev_first = si.flags & kTileFirst;
      prev_ord = cur_ord;
    }
    if (ok && j >= 1) issue_pv(j - 1, prev_first, prev_ord);
    commit(mma_done);  // completes when every MMA issued above has finished
    wait_all(mma_done, 0);
  } else {
    // ---------------------------------------------------- softmax / epilogue
    // warp w serves heads 16 w .. 16 w + 15 (TMEM lanes 32 w .. 32 w + 15):
    // the quad of lanes 4 g .. 4 g + 3 holds heads ra = 16 w + g and
    // rb = ra + 8, each thread keys 8 i + 2 (lane % 4) + {0, 1} of a tile
    const int t = threadIdx.x;
    const int g = lane >> 2, qi = lane & 3;
    const int ra = warp * 16 + g, rb = ra + 8;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* prow_a = smem + C::kPOff + ra * 128;
    uint8_t* prow_b = smem + C::kPOff + rb * 128;
    const float sl2 = p.scale_log2;
    const bool pos_scale = sl2 > 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    ItemCoord c{};
    for (int j = 0;; ++j) {
      const int s = j % C::kStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&kv_full[s], (j / C::kStages) & 1))) break;
      const StageInfo si = info[s];
      if (si.item < 0) break;
      const bool first = si.flags & kTileFirst;
      if (first) {
        c = item_coord_n(p, si.item, kWideHeads);
        m_a = m_b = -INFINITY;
        l_a = l_b = 0.f;
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      float x[64];
      tmem_ld_16x256b_x16(lane_addr + C::kSCol + (uint32_t)((j & 1) * kWideKeys), x);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[j & 1]);

      uint32_t pa[16], pb[16];
      float alpha_a, alpha_b;
      if (pos_scale)
        wide_softmax_tile<true>(x, si.rows, qi, sl2, m_a, m_b, l_a, l_b, pa, pb, alpha_a, alpha_b);
      else
        wide_softmax_tile<false>(x, si.rows, qi, sl2, m_a, m_b, l_a, l_b, pa, pb, alpha_a, alpha_b);
      // the P buffer and O are free once the previous tile's PV has finished
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (j - 1) & 1))) break;
        tc_fence_after();
      }
      // a head whose maximum moved (never on an item's first tile, where PV overwrites O)
      if (__any_sync(0xffffffffu, !first && (alpha_a != 1.f || alpha_b != 1.f))) {
        float o[32];
#pragma unroll 1
        for (int cb = 0; cb < D; cb += 64) {
          tmem_ld_16x256b_x8(lane_addr + C::kOCol + cb, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            o[4 * i] *= alpha_a;
            o[4 * i + 1] *= alpha_a;
            o[4 * i + 2] *= alpha_b;
            o[4 * i + 3] *= alpha_b;
          }
          tmem_st_16x256b_x8(lane_addr + C::kOCol + cb, o);
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
      // P rows, K-major with the 128-byte swizzle: keys 8 i .. 8 i + 7 form 16-byte chunk i
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t off = (uint32_t)((i >> 3) * C::kPHalf) + ((((uint32_t)(i & 7)) ^ (uint32_t)g) << 4) + 4u * qi;
        *reinterpret_cast<uint32_t*>(prow_a + off) = pa[i];
        *reinterpret_cast<uint32_t*>(prow_b + off) = pb[i];
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(p_full);

      if (si.flags & kTileLast) {
        // ---- item epilogue: O / l -> out (one split) or the split's partial
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, j & 1))) break;
        tc_fence_after();
        float o[64];
        tmem_ld_16x256b_x16(lane_addr + C::kOCol, o);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(o_free);
        float la = l_a, lb = l_b;
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
          la += __shfl_xor_sync(0xffffffffu, la, off);
          lb += __shfl_xor_sync(0xffffffffu, lb, off);
        }
        if (si.flags & kUnitSingleSplit) {
          const float ia = 1.f / la, ib = 1.f / lb;
          __nv_bfloat16* oa = static_cast<__nv_bfloat16*>(p.out) + ((size_t)c.b * p.H + c.h0 + ra) * D + 2 * qi;
          __nv_bfloat16* ob = oa + 8 * D;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            *reinterpret_cast<uint32_t*>(oa + 8 * i) = pack_bf16x2(o[4 * i] * ia, o[4 * i + 1] * ia);
            *reinterpret_cast<uint32_t*>(ob + 8 * i) = pack_bf16x2(o[4 * i + 2] * ib, o[4 * i + 3] * ib);
          }
        } else {
          const size_t part = ((size_t)c.unit * p.nsplit + c.split) * p.G + (size_t)c.hsl * kWideHeads + ra;
          float* da = p.ws_o + part * D + 2 * qi;
          float* db = da + 8 * D;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            *reinterpret_cast<float2*>(da + 8 * i) = make_float2(o[4 * i], o[4 * i + 1]);
            *reinterpret_cast<float2*>(db + 8 * i) = make_float2(o[4 * i + 2], o[4 * i + 3]);
          }
          if (qi == 0) {
            p.ws_ml[part] = make_float2(m_a, la);
            p.ws_ml[part + 8] = make_float2(m_b, lb);
          }
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
