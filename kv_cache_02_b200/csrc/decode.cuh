// GQA decode over a KV cache.
//
// Every K/V row is brought from HBM once by TMA and serves all of its group's
// query heads ("GQA 完全拆解", section 工程实现: the group's query heads share
// one thread block and one load of each KV block).
//
// bf16 path. A CTA has 5 warps: warp 4 is the TMA producer (64-key tiles of K
// and V, 128-byte swizzled, in a ring of mbarrier-guarded stages); warps 0..3
// each own 16 keys of every tile and run on the tensor cores:
//     S^T[16 keys x 8 heads]  = K[16 x d] * Q^T[d x 8]        (mma.sync m16n8k16)
//     online softmax over keys, per head, in fp32 (log2 domain)
//     O^T[d x 8 heads]       += V^T[d x 16 keys] * P^T[16 x 8]
// Keys sit in the MMA M dimension and up to 8 of the group's heads in N, so
// G = 8 fills the instruction and G = 4 uses half of it. P^T comes from the
// S^T accumulator through movmatrix (a register transpose). At the end of a
// (b, g) unit the four warps' (m, l, O) are merged in shared memory.
//
// The key axis of each (b, g) unit is cut into splits of `chunk` keys; a
// work item is (b, g, split, head slice). bf16: persistent CTAs, two per SM;
// each CTA's producer takes items from a tagged atomic counter, split-major
// (split s of every unit before split s + 1), and streams their tiles
// through its ring without a break, so a work item's epilogue (merging the
// four warps, writing the output or the split's partial) overlaps the next
// item's loads, and late items go to whichever CTA is free. The counter word
// carries a per-call tag next to the count, so stale or uninitialised
// workspace contents read as "no items taken yet": the workspace needs no
// initialisation; the last CTA out resets it, so a CUDA graph replay, which
// repeats the tag, finds it unclaimed. Units with more than one split are
// merged by decode_combine_kernel (log-sum-exp), launched as a programmatic
// dependent so that its launch overlaps the decode kernel.
//
// Paged caches: the producer is the whole warp (table entries loaded
// together, one lane per 16-row box). 8-bit caches: the consumers turn codes
// into fp16 and take 32 keys of alternate tiles each (warp_tile_i8).
//
// f32 path (float32 storage, small problems): plain FMA, one warp per head.
#pragma once

#include "common.cuh"

namespace gqa {

constexpr int kDecTileKeys = 64;
constexpr int kDecConsumerWarps = 4;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecBoxRows = 16;  // TMA box height; the ragged tail is read in 16-row steps
constexpr int kDecHeadsPerCta = 8;

// Ring stage geometry. bf16 cache: K tile then V tile, each in 128-byte
// column boxes. 8-bit cache (kInt8, d = 128): a key row of codes is one
// 128-byte swizzled row; K codes, V codes, then the tile's 64 K scales and
// 64 V scales (float), the stage rounded up to 1024 bytes.
template <int D, bool kInt8 = false>
struct DecCfg {
  static_assert(!kInt8 || D == 128, "the 8-bit cache is laid out for head dim 128");
  static constexpr int kElt = kInt8 ? 1 : 2;
  static constexpr int kHalves = D * kElt / 128;               // 128-byte column boxes per row
  static constexpr int kHalfBytes = kDecTileKeys * 128;        // one column box of a tile
  static constexpr int kTileBytes = kDecTileKeys * D * kElt;   // K (or V) tile
  static constexpr int kScaleOff = 2 * kTileBytes;             // 8-bit: K scales, then V scales
  static constexpr int kQOff = kScaleOff + 2 * kDecTileKeys * 4;  // 8-bit: the item's q rows (first tile)
  static constexpr int kStages = kInt8 ? 5 : ((D == 128) ? 3 : 6);
  static constexpr int kStageBytes = kInt8 ? (kQOff + kDecHeadsPerCta * D * 2 + 1023) / 1024 * 1024
                                           : 2 * kTileBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // merge scratch: per consumer warp, m and l of 8 heads, then O of 8 heads
  static constexpr int kMergeFloats = kDecConsumerWarps * (2 * kDecHeadsPerCta + kDecHeadsPerCta * D);
  // persistent kernel: ring, then merge/combine scratch (the ring keeps
  // streaming while a work item's epilogue runs), stage records, barriers
  static constexpr int kMergeOff = kRingBytes;
  static constexpr int kInfoOff = kMergeOff + kMergeFloats * 4;
  static constexpr int kBarOff = kInfoOff + kStages * 16;
  static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8;
};

struct DecodeParams {
  const void* q;
  void* out;
  float* ws_o;                 // [B*K*nsplit*G, D] partial O (unnormalised, relative to m)
  float2* ws_ml;               // [B*K*nsplit*G] partial (m, l), m in log2 units
  // fused append (gqa_decode_append): seqlens holds pos, lengths are pos + len_add
  const void* k_new;           // [B, K, D] or null
  const void* v_new;
  void* k_cache_w;             // the caches, written at row pos[b]
  void* v_cache_w;
  int len_add;                 // 0 (decode) or 1 (decode after append)
  unsigned long long* ws_queue;  // [2]: work-item counter of the persistent kernel and its exit counter (tag | count)
  int nitems;                  // B * K * nsplit * hslices
  const int32_t* seqlens;
  int B, H, K, S_max, G, hslices, chunk, nsplit;
  // paged cache (gqa_decode_paged): null for the contiguous cache
  // [B, K, S_max, D]; otherwise the cache is a pool of num_blocks blocks
  // [K, block_size, D] and block_table[b * max_blocks + i] is the block that
  // holds keys i * block_size .. (i + 1) * block_size - 1 of sequence b
  // (S_max = max_blocks * block_size). The TMA maps view either as rows of D.
  const int32_t* block_table;
  int max_blocks, block_size, num_blocks;
  unsigned long long tag;      // 40-bit, nonzero, different on every call
  float scale_log2;            // scale * log2(e)
};

constexpr int kCntBits = 24;              // count field of a tagged counter (work items stay below 2^24)
constexpr int kMaxCombineSplits = 1024;  // most splits per unit that a decode plan makes

__device__ __forceinline__ unsigned long long atom_add_relaxed(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.add.relaxed.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long atom_cas_relaxed(unsigned long long* p, unsigned long long cmp,
                                                               unsigned long long val) {
  unsigned long long old;
  asm volatile("atom.cas.relaxed.gpu.global.b64 %0, [%1], %2, %3;" : "=l"(old) : "l"(p), "l"(cmp), "l"(val)
               : "memory");
  return old;
}

// Take a ticket from a tagged counter: returns 1, 2, 3, ... in the order the
// CTAs of the current call arrive. A word whose tag differs from the call's
// tag counts as zero: the first arrival claims it with one compare-and-swap,
// every later one adds to the count (the tag, in the high bits, is left
// alone). Nothing ever waits for another CTA.
__device__ __forceinline__ int take_ticket(unsigned long long* cnt, unsigned long long tag) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(cnt);
  for (int attempt = 0; attempt < 64; ++attempt) {
    if ((cur >> kCntBits) == tag) return (int)((atom_add_relaxed(cnt, 1ull) & ((1ull << kCntBits) - 1)) + 1);
    const unsigned long long prev = atom_cas_relaxed(cnt, cur, (tag << kCntBits) | 1ull);
    if (prev == cur) return 1;
    cur = prev;  // another CTA claimed it first (or the word changed): look again
  }
  raise_error(GQA_DEVERR_TIMEOUT);
  return 0;
}

// Called once per CTA after its last ticket (q[0] the counter, q[1] an exit
// counter of the same kind): the last CTA out resets both words to tag 0,
// which no call uses (call tags are odd), so that a launch that repeats its
// tag -- a CUDA graph replay -- finds them unclaimed. The fences order every
// CTA's tickets before its exit ticket, and all of them before the reset.
__device__ __forceinline__ void leave_queue(unsigned long long* q, unsigned long long tag) {
  __threadfence();
  if (take_ticket(q + 1, tag) == (int)gridDim.x) {
    __threadfence();
    reinterpret_cast<volatile unsigned long long*>(q)[0] = 0ull;
    reinterpret_cast<volatile unsigned long long*>(q)[1] = 0ull;
  }
}

// Row of key t of KV head g in the [rows, D] view of a paged pool, key t
// being in block blk (a table entry: outside [0, num_blocks) it sets
// GQA_DEVERR_BLOCK and block 0 is used).
__device__ __forceinline__ int paged_row(const DecodeParams& p, int blk, int g, int t) {
  if ((unsigned)blk >= (unsigned)p.num_blocks) {
    raise_error(GQA_DEVERR_BLOCK);
    blk = 0;
  }
  return (blk * p.K + g) * p.block_size + t % p.block_size;
}

// Row of key t of unit (b, g) in the [rows, D] view of the cache (kPaged
// false) or the pool. A table entry outside [0, num_blocks) sets
// GQA_DEVERR_BLOCK and reads block 0. Paging is a template parameter of the
// kernels, so the contiguous kernels carry none of the paged code.
template <bool kPaged>
__device__ __forceinline__ int kv_row(const DecodeParams& p, int b, int g, int t) {
  if constexpr (!kPaged) return (b * p.K + g) * p.S_max + t;
  return paged_row(p, __ldg(p.block_table + (size_t)b * p.max_blocks + t / p.block_size), g, t);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
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

__device__ __forceinline__ int valid_len(int len, int S_max) { return (len < 0 || len > S_max) ? 0 : len; }

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");
}

// ---------------------------------------------------------------------------
// pieces shared by the bf16 kernels

// TMA loads of one tile (rows of K and V of one unit) into ring stage `s`.
// TMA loads of one tile into a ring stage: a full tile as one 64-row box per
// 128-byte column half (tm_*64), a partial one as 16-row boxes (tm_*16). The
// 128-byte swizzle repeats every 8 rows, so both land in the same layout.
// The producer is one thread; fewer, larger boxes keep it ahead of the ring.
template <int D>
__device__ __forceinline__ void issue_tile(uint8_t* stage, uint64_t* full, const CUtensorMap* tm_k64,
                                           const CUtensorMap* tm_v64, const CUtensorMap* tm_k16,
                                           const CUtensorMap* tm_v16, int row0, int rows, uint64_t policy) {
  using C = DecCfg<D>;
  if (rows == kDecTileKeys) {
    mbar_arrive_expect_tx(full, (uint32_t)(kDecTileKeys * 128 * C::kHalves * 2));
#pragma unroll
    for (int hf = 0; hf < C::kHalves; ++hf) {
      tma_load_2d(stage + hf * C::kHalfBytes, tm_k64, hf * 64, row0, full, policy);
      tma_load_2d(stage + C::kTileBytes + hf * C::kHalfBytes, tm_v64, hf * 64, row0, full, policy);
    }
    return;
  }
  const int nbox = (rows + kDecBoxRows - 1) / kDecBoxRows;
  mbar_arrive_expect_tx(full, (uint32_t)(nbox * kDecBoxRows * 128 * C::kHalves * 2));
  for (int bx = 0; bx < nbox; ++bx) {
#pragma unroll
    for (int hf = 0; hf < C::kHalves; ++hf) {
      const int off = hf * C::kHalfBytes + bx * kDecBoxRows * 128;
      tma_load_2d(stage + off, tm_k16, hf * 64, row0 + bx * kDecBoxRows, full, policy);
      tma_load_2d(stage + C::kTileBytes + off, tm_v16, hf * 64, row0 + bx * kDecBoxRows, full, policy);
    }
  }
}

// The 8-bit cache: the codes of a full tile as one 64-row box each for K and
// V, a partial tile as 16-row boxes; the tile's 64 K and 64 V scales as one
// box each from the [units, S_max] scale arrays (a box reaching past a row's
// end reads the next unit's scales, past the array's end TMA fills zeros;
// only scales of valid keys are used).
template <int D>
__device__ __forceinline__ void issue_tile_i8(uint8_t* stage, uint64_t* full, const CUtensorMap* tm_k64,
                                              const CUtensorMap* tm_v64, const CUtensorMap* tm_k16,
                                              const CUtensorMap* tm_v16, const CUtensorMap* tm_ks,
                                              const CUtensorMap* tm_vs, int row0, int unit, int t0, int rows,
                                              const void* q_rows, uint32_t q_bytes, uint64_t policy) {
  using C = DecCfg<D, true>;
  constexpr uint32_t kScaleBytes = kDecTileKeys * 4;
  if (rows == kDecTileKeys) {
    mbar_arrive_expect_tx(full, (uint32_t)(2 * C::kTileBytes) + 2 * kScaleBytes + q_bytes);
    tma_load_2d(stage, tm_k64, 0, row0, full, policy);
    tma_load_2d(stage + C::kTileBytes, tm_v64, 0, row0, full, policy);
  } else {
    const int nbox = (rows + kDecBoxRows - 1) / kDecBoxRows;
    mbar_arrive_expect_tx(full, (uint32_t)(nbox * kDecBoxRows * 128 * 2) + 2 * kScaleBytes + q_bytes);
    for (int bx = 0; bx < nbox; ++bx) {
      tma_load_2d(stage + bx * kDecBoxRows * 128, tm_k16, 0, row0 + bx * kDecBoxRows, full, policy);
      tma_load_2d(stage + C::kTileBytes + bx * kDecBoxRows * 128, tm_v16, 0, row0 + bx * kDecBoxRows, full, policy);
    }
  }
  tma_load_2d(stage + C::kScaleOff, tm_ks, t0, unit, full, policy);
  tma_load_2d(stage + C::kScaleOff + kScaleBytes, tm_vs, t0, unit, full, policy);
  if (q_bytes) bulk_load(stage + C::kQOff, q_rows, q_bytes, full);
}

// Q^T as the fp16 B operand of the 8-bit path, from the item's q rows in
// shared memory: in the 16-dim step ks the lane holds head lane/4, dims
// 16 ks + 4 (lane%4) + {0, 1} (b0) and + {2, 3} (b1) -- the order in which a
// key row's codes reach the A operand (warp_tile_i8), so the dot products
// are unchanged.
template <int D>
__device__ __forceinline__ void load_q_frag_i8(uint32_t (&qf)[D / 16][2], const __nv_bfloat16* q, int lane, int nh) {
  const int hn = lane >> 2;
  const bool hv = hn < nh;
  const uint2* qrow = reinterpret_cast<const uint2*>(q + (size_t)(hv ? hn : 0) * D);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint2 w = qrow[ks * 4 + (lane & 3)];
    const float f0 = __uint_as_float(w.x << 16), f1 = __uint_as_float(w.x & 0xffff0000u);
    const float f2 = __uint_as_float(w.y << 16), f3 = __uint_as_float(w.y & 0xffff0000u);
    qf[ks][0] = hv ? pack_f16x2(f0, f1) : 0u;
    qf[ks][1] = hv ? pack_f16x2(f2, f3) : 0u;
  }
}

// Q^T as the B operand (k = dims, n = heads): lane holds head lane/4, dims
// 2*(lane%4) + {0,1} (b0) and + 8 (b1) of every 16-dim step.
template <int D>
__device__ __forceinline__ void load_q_frag(uint32_t (&qf)[D / 16][2], const __nv_bfloat16* q, int lane, int nh) {
  const int hn = lane >> 2;
  const bool hv = hn < nh;
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(q + (size_t)(hv ? hn : 0) * D);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t lo = __ldg(qrow + ks * 8 + (lane & 3));
    const uint32_t hi = __ldg(qrow + ks * 8 + 4 + (lane & 3));
    qf[ks][0] = hv ? lo : 0u;
    qf[ks][1] = hv ? hi : 0u;
  }
}

// Running softmax state of one consumer warp for heads a = 2*(lane%4) and
// b = a + 1 over the keys it has seen (log2 units).
template <int D>
struct WarpState {
  float m_a, m_b, l_a, l_b;
  float b_a, b_b;  // 8-bit path: sum of the fp16 P^T entries, the weight of the code bias in o
  float o[D / 16][4];
  __device__ __forceinline__ void reset() {
    m_a = m_b = -INFINITY;
    l_a = l_b = 0.f;
    b_a = b_b = 0.f;
#pragma unroll
    for (int md = 0; md < D / 16; ++md) o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;
  }
};

// One warp's 16 keys (kb .. kb+15) of the tile in `stage`; `rows` keys of the
// tile are valid (the rest may hold anything, NaN included).
template <int D>
__device__ __forceinline__ void warp_tile(WarpState<D>& st, const uint32_t (&qf)[D / 16][2], uint32_t stage_addr,
                                          int kb, int rows, int lane, float scale_log2) {
  using C = DecCfg<D>;
  const uint32_t k_base = stage_addr;
  const uint32_t v_base = stage_addr + C::kTileBytes;
  // ldmatrix row/column assignment (lane -> 8x8 matrix lane/8)
  const int k_row = kb + (lane & 7) + ((lane >> 3) & 1) * 8;  // K: (r0-7,c0-7) (r8-15,c0-7) (r0-7,c8-15) ...
  const int k_col8 = lane >> 4;
  const int v_row = kb + (lane & 7) + (lane >> 4) * 8;  // V^T: (d0-7,k0-7) (d8-15,k0-7) (d0-7,k8-15) ...
  const int v_col8 = (lane >> 3) & 1;

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
  const float x0 = v0 ? c[0] * scale_log2 : -INFINITY;
  const float x1 = v0 ? c[1] * scale_log2 : -INFINITY;
  const float x2 = v1 ? c[2] * scale_log2 : -INFINITY;
  const float x3 = v1 ? c[3] * scale_log2 : -INFINITY;
  float mx_a = fmaxf(x0, x2), mx_b = fmaxf(x1, x3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
  }
  const float mn_a = fmaxf(st.m_a, mx_a), mn_b = fmaxf(st.m_b, mx_b);
  const float al_a = fast_exp2(st.m_a - mn_a), al_b = fast_exp2(st.m_b - mn_b);
  st.m_a = mn_a;
  st.m_b = mn_b;
  const float p0 = fast_exp2(x0 - mn_a), p1 = fast_exp2(x1 - mn_b);
  const float p2 = fast_exp2(x2 - mn_a), p3 = fast_exp2(x3 - mn_b);
  st.l_a = st.l_a * al_a + p0 + p2;
  st.l_b = st.l_b * al_b + p1 + p3;
#pragma unroll
  for (int md = 0; md < D / 16; ++md) {
    st.o[md][0] *= al_a;
    st.o[md][1] *= al_b;
    st.o[md][2] *= al_a;
    st.o[md][3] *= al_b;
  }

  // P^T (k = keys, n = heads) from the S^T accumulator layout
  const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
  const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));

  // keys of this block past the valid rows: zero their V^T entries
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
    mma_bf16_16816(st.o[md], a0 & mask_lo, a1 & mask_lo, a2 & mask_hi, a3 & mask_hi, pb0, pb1);
  }
}

// The 8-bit cache. Codes reach the MMAs as exact fp16 values biased by
// kCodeBias (code + 1152: the fp16 with bits 0x64uu is 1024 + u for a byte u =
// code + 128), fp16 x fp16 -> fp32; the bias is taken out of the sums
// afterwards (one subtraction per score, one per output element) rather than
// out of every code. The K scale multiplies the score and the V scale the
// probability (the softmax sums stay unscaled).
//   Q K^T: a plain ldmatrix gives a lane 4 consecutive codes of one key row,
// the A operand with the head dims permuted as in load_q_frag_i8; the score
// of key k for head h is S - kCodeBias * sum_d q_hd.
//   V^T P^T: a transposing ldmatrix gives a lane the codes of dims 2g, 2g+1
// for keys 2t, 2t+1 (g = lane/4, t = lane%4), so byte selects alone make the
// A operand, row g of a 16-dim step d0 being dim d0 + 2g and row g + 8 dim
// d0 + 2g + 1 (see stash_warp_state); o then holds O + kCodeBias * sum_k P_k.
constexpr float kCodeBias = 1152.f;

// kCodeBias * sum_d q_hd for this lane's score heads a = 2*(lane%4) and
// b = a + 1, from the fp16 Q fragment of load_q_frag_i8 (the values the MMA
// multiplies).
template <int D>
__device__ __forceinline__ void q_code_bias(const uint32_t (&qf)[D / 16][2], int lane, float& qb_a, float& qb_b) {
  float sum = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&qf[ks][r]));
      sum += f.x + f.y;
    }
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);  // the four lanes of head lane/4
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  qb_a = kCodeBias * __shfl_sync(0xffffffffu, sum, 8 * (lane & 3));
  qb_b = kCodeBias * __shfl_sync(0xffffffffu, sum, 8 * (lane & 3) + 4);
}

// One warp's NB x 16 keys (kb .. kb + 16 NB - 1) of the 8-bit tile in
// `stage`: NB independent 16-key blocks, so that NB MMA chains are in
// flight; `rows` keys of the tile are valid, kb < rows.
template <int D, int NB>
__device__ __forceinline__ void warp_tile_i8(WarpState<D>& st, const uint32_t (&qf)[D / 16][2], float qb_a,
                                             float qb_b, uint32_t stage_addr, const float* sk, const float* sv,
                                             int kb, int rows, int lane, float scale_log2) {
  static_assert(NB == 1 || NB == 2, "one or two key blocks");
  using C = DecCfg<D, true>;
  const uint32_t k_base = stage_addr;
  const uint32_t v_base = stage_addr + C::kTileBytes;
  // ldmatrix: matrices (rows 0-7, chunk c) (rows 8-15, chunk c) (rows 0-7, chunk c+1) (rows 8-15, chunk c+1)
  const int row = kb + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int ch = lane >> 4;

  // S^T + bias = K * Q^T for each block, two 16-dim steps per ldmatrix
  float c[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
#pragma unroll
  for (int j = 0; j < D / 32; ++j) {
    uint32_t r[NB][4], lo[NB][4], hi[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      ldmatrix_x4(k_base + sw128(row + 16 * nb, 2 * j + ch), r[nb][0], r[nb][1], r[nb][2], r[nb][3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) codes4_to_f16x2_biased(r[nb][i], lo[nb][i], hi[nb][i]);
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
      mma_f16_16816(c[nb], lo[nb][0], lo[nb][1], hi[nb][0], hi[nb][1], qf[2 * j][0], qf[2 * j][1]);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
      mma_f16_16816(c[nb], lo[nb][2], lo[nb][3], hi[nb][2], hi[nb][3], qf[2 * j + 1][0], qf[2 * j + 1][1]);
  }

  // online softmax over the keys: key kb + lane/4 + 8 i for i < 2 NB (block
  // i/2, accumulator entries c0/c1 for even i and c2/c3 for odd i), each
  // score unbiased and scaled by its key's K scale
  constexpr int NK = 2 * NB;
  const int key0 = kb + (lane >> 2);
  bool vk[NK];
  float xa[NK], xb[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    vk[i] = key0 + 8 * i < rows;
    const float sc = vk[i] ? sk[key0 + 8 * i] * scale_log2 : 0.f;
    xa[i] = vk[i] ? (c[i >> 1][2 * (i & 1)] - qb_a) * sc : -INFINITY;
    xb[i] = vk[i] ? (c[i >> 1][2 * (i & 1) + 1] - qb_b) * sc : -INFINITY;
  }
  float mx_a = fmaxf(xa[0], xa[1]), mx_b = fmaxf(xb[0], xb[1]);
  if constexpr (NB == 2) {
    mx_a = fmaxf(mx_a, fmaxf(xa[2], xa[3]));
    mx_b = fmaxf(mx_b, fmaxf(xb[2], xb[3]));
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
  }
  const float mn_a = fmaxf(st.m_a, mx_a), mn_b = fmaxf(st.m_b, mx_b);
  const float al_a = fast_exp2(st.m_a - mn_a), al_b = fast_exp2(st.m_b - mn_b);
  st.m_a = mn_a;
  st.m_b = mn_b;
  float pa[NK], pb[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    pa[i] = fast_exp2(xa[i] - mn_a);
    pb[i] = fast_exp2(xb[i] - mn_b);
  }
  float sa = pa[0] + pa[1], sb = pb[0] + pb[1];
  if constexpr (NB == 2) {
    sa += pa[2] + pa[3];
    sb += pb[2] + pb[3];
  }
  st.l_a = st.l_a * al_a + sa;
  st.l_b = st.l_b * al_b + sb;
#pragma unroll
  for (int md = 0; md < D / 16; ++md) {
    st.o[md][0] *= al_a;
    st.o[md][1] *= al_b;
    st.o[md][2] *= al_a;
    st.o[md][3] *= al_b;
  }

  // P^T times the V scales (keys past the valid rows: 0, their scales are
  // never read), and the sums of those fp16 entries for the bias
  uint32_t pt[NK];
  float bs_a = 0.f, bs_b = 0.f;
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const float w = vk[i] ? sv[key0 + 8 * i] : 0.f;
    const uint32_t pk = pack_f16x2(pa[i] * w, pb[i] * w);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&pk));
    bs_a += f.x;
    bs_b += f.y;
    pt[i] = movmatrix_trans(pk);
  }
  st.b_a = st.b_a * al_a + bs_a;
  st.b_b = st.b_b * al_b + bs_b;

  // O^T + bias = V^T * P^T for each block, two 16-dim steps per ldmatrix:
  // r[0]/r[1] keys 0-7 / 8-15 of the block for the dims of step 2j, r[2]/r[3] of step 2j + 1
#pragma unroll
  for (int j = 0; j < D / 32; ++j) {
    uint32_t r[NB][4], ev[NB][4], od[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      ldmatrix_x4_trans(v_base + sw128(row + 16 * nb, 2 * j + ch), r[nb][0], r[nb][1], r[nb][2], r[nb][3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) code_pairs_to_f16x2_biased(r[nb][i], ev[nb][i], od[nb][i]);
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      mma_f16_16816(st.o[2 * j], ev[nb][0], od[nb][0], ev[nb][1], od[nb][1], pt[2 * nb], pt[2 * nb + 1]);
      mma_f16_16816(st.o[2 * j + 1], ev[nb][2], od[nb][2], ev[nb][3], od[nb][3], pt[2 * nb], pt[2 * nb + 1]);
    }
  }
}

// Write one warp's state into the merge scratch (after a consumer barrier).
template <int D, bool kInt8 = false>
__device__ __forceinline__ void stash_warp_state(float* merge, const WarpState<D>& st, int warp, int lane) {
  float* red_m = merge;
  float* red_l = red_m + kDecConsumerWarps * kDecHeadsPerCta;
  float* ow = red_l + kDecConsumerWarps * kDecHeadsPerCta + warp * kDecHeadsPerCta * D;
  float l_a = st.l_a, l_b = st.l_b;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
  }
  const int ha = 2 * (lane & 3);
  if (lane < 4) {
    red_m[warp * 8 + ha] = st.m_a;
    red_m[warp * 8 + ha + 1] = st.m_b;
    red_l[warp * 8 + ha] = l_a;
    red_l[warp * 8 + ha + 1] = l_b;
  }
  // accumulator rows g and g + 8 of a 16-dim step: dims g and g + 8, or for
  // the 8-bit path dims 2g and 2g + 1, less the code bias times the P^T sums
  const int dr = lane >> 2;
  const int da = kInt8 ? 2 * dr : dr, db = kInt8 ? 2 * dr + 1 : dr + 8;
  if constexpr (kInt8) {
    float b_a = st.b_a, b_b = st.b_b;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      b_a += __shfl_xor_sync(0xffffffffu, b_a, off);
      b_b += __shfl_xor_sync(0xffffffffu, b_b, off);
    }
    const float c_a = kCodeBias * b_a, c_b = kCodeBias * b_b;
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      ow[ha * D + md * 16 + da] = st.o[md][0] - c_a;
      ow[(ha + 1) * D + md * 16 + da] = st.o[md][1] - c_b;
      ow[ha * D + md * 16 + db] = st.o[md][2] - c_a;
      ow[(ha + 1) * D + md * 16 + db] = st.o[md][3] - c_b;
    }
  } else {
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      ow[ha * D + md * 16 + da] = st.o[md][0];
      ow[(ha + 1) * D + md * 16 + da] = st.o[md][1];
      ow[ha * D + md * 16 + db] = st.o[md][2];
      ow[(ha + 1) * D + md * 16 + db] = st.o[md][3];
    }
  }
}

// Merge the four warps' states for output (h, dim): returns (M, L, O).
template <int D>
__device__ __forceinline__ void merged(const float* merge, int h, int dim, float& M, float& L, float& O) {
  const float* red_m = merge;
  const float* red_l = red_m + kDecConsumerWarps * kDecHeadsPerCta;
  const float* red_o = red_l + kDecConsumerWarps * kDecHeadsPerCta;
  M = -INFINITY;
#pragma unroll
  for (int ww = 0; ww < kDecConsumerWarps; ++ww) M = fmaxf(M, red_m[ww * 8 + h]);
  L = 0.f;
  O = 0.f;
#pragma unroll
  for (int ww = 0; ww < kDecConsumerWarps; ++ww) {
    const float f = fast_exp2(red_m[ww * 8 + h] - M);
    L += red_l[ww * 8 + h] * f;
    O += red_o[(ww * kDecHeadsPerCta + h) * D + dim] * f;
  }
}

// ---------------------------------------------------------------------------
// fixed splits: one CTA per (b, g, split, head slice)

struct DecItem {
  int b, g, unit, split, hsl, len, t_begin, t_end, h0, nh;
};

// Work item -> (unit, split, head slice); head slice varies fastest so the
// CTAs that read the same KV chunk for different head slices run together.
__device__ __forceinline__ DecItem decode_item(const DecodeParams& p, int heads_per_cta) {
  DecItem it;
  const int item = blockIdx.x;
  it.hsl = item % p.hslices;
  const int rest = item / p.hslices;
  it.split = rest % p.nsplit;
  it.unit = rest / p.nsplit;
  it.b = it.unit / p.K;
  it.g = it.unit % p.K;
  int len = __ldg(p.seqlens + it.b) + p.len_add;
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

// ---------------------------------------------------------------------------
// bf16: persistent CTAs (two per SM). The producer thread takes work items
// (unit, split, head slice) from a tagged atomic counter in unit order and
// streams their tiles through the ring without a break; a 16-byte record per
// stage tells the consumers which item a tile belongs to and whether it is
// the item's first or last. A consumer epilogue (warp merge, output or
// partial, arrival, combine) overlaps the loads of the next item.

constexpr int kTileFirst = 1;        // the first tile of a work item
constexpr int kTileLast = 2;         // the last tile of a work item
constexpr int kUnitSingleSplit = 4;  // the item's unit has one split: its output is final

struct StageInfo {
  int item;     // work item, or -1: no more work
  int rows;     // valid keys in the tile
  int flags;    // kTileFirst | kTileLast | kUnitSingleSplit
  int new_row;  // row of the tile that holds the appended token, or -1
};

struct ItemCoord {
  int b, g, unit, split, hsl, h0, nh;
};

__device__ __forceinline__ ItemCoord item_coord_n(const DecodeParams& p, int item, int heads_per_cta) {
  ItemCoord c;
  c.hsl = item % p.hslices;
  const int rest = item / p.hslices;
  c.unit = rest % (p.B * p.K);  // split-major: the short last splits of the units come last
  c.split = rest / (p.B * p.K);
  c.b = c.unit / p.K;
  c.g = c.unit % p.K;
  c.h0 = c.g * p.G + c.hsl * heads_per_cta;
  c.nh = min(heads_per_cta, p.G - c.hsl * heads_per_cta);
  return c;
}

__device__ __forceinline__ ItemCoord item_coord(const DecodeParams& p, int item) {
  ItemCoord c;
  c.hsl = item % p.hslices;
  const int rest = item / p.hslices;
  c.unit = rest % (p.B * p.K);  // split-major: the short last splits of the units come last
  c.split = rest / (p.B * p.K);
  c.b = c.unit / p.K;
  c.g = c.unit % p.K;
  c.h0 = c.g * p.G + c.hsl * kDecHeadsPerCta;
  c.nh = min(kDecHeadsPerCta, p.G - c.hsl * kDecHeadsPerCta);
  return c;
}

// End of a work item: merge the four warps, then write the output (a unit
// with a single split) or the split's partial for decode_combine_kernel.
template <int D, bool kInt8 = false>
__device__ __forceinline__ void item_epilogue(const DecodeParams& p, const ItemCoord& c, const WarpState<D>& st,
                                              float* merge, bool single, int tid, int warp, int lane) {
  __nv_bfloat16* out_row = static_cast<__nv_bfloat16*>(p.out) + ((size_t)c.b * p.H + c.h0) * D;
  consumer_bar();  // the previous epilogue has finished with the scratch
  stash_warp_state<D, kInt8>(merge, st, warp, lane);
  consumer_bar();
  const size_t part = ((size_t)c.unit * p.nsplit + c.split) * p.G + (size_t)c.hsl * kDecHeadsPerCta;
  for (int i = tid; i < c.nh * D; i += kDecConsumerWarps * 32) {
    const int h = i / D, dim = i % D;
    float M, L, O;
    merged<D>(merge, h, dim, M, L, O);
    if (single) {
      out_row[i] = __float2bfloat16_rn(O / L);
    } else {
      p.ws_o[(part + h) * D + dim] = O;
      if (dim == 0) p.ws_ml[part + h] = make_float2(M, L);
    }
  }
}

// The appended token (gqa_decode_append): its K and V replace row `r` of the
// tile just landed in shared memory (one warp, one 16-byte chunk per lane)
// and are written to the cache at that row. The tile's rows are cache rows
// t0 .. t0+rows-1, so row r is cache row len-1 = pos.
template <int D, bool kPaged>
__device__ __forceinline__ void append_row(const DecodeParams& p, const ItemCoord& c, uint8_t* stage, int r,
                                           int lane) {
  using C = DecCfg<D>;
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  const int pos = __ldg(p.seqlens + c.b);
  if (lane < 2 * kChunks) {
    const bool is_v = lane >= kChunks;
    const int ch = is_v ? lane - kChunks : lane;
    const size_t row = (size_t)c.b * p.K + c.g;  // unit (b, g)
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(
                                static_cast<const __nv_bfloat16*>(is_v ? p.v_new : p.k_new) + row * D) + ch);
    uint8_t* dst = stage + (is_v ? C::kTileBytes : 0) + (ch >> 3) * C::kHalfBytes + sw128((uint32_t)r, ch & 7);
    *reinterpret_cast<uint4*>(dst) = val;
    if (c.hsl == 0) {  // one head slice writes the cache
      __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(is_v ? p.v_cache_w : p.k_cache_w);
      reinterpret_cast<uint4*>(cache + (size_t)kv_row<kPaged>(p, c.b, c.g, pos) * D)[ch] = val;
    }
  }
  // the stage is refilled by TMA (async proxy) once released: order these writes first
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
}

// Producer of the paged kernel: the whole warp. Lane 0 takes the tickets
// and the stage waits; at an item's start the lanes load up to 32 of its
// table entries at once (one coalesced load, lane j block j of the window),
// and each tile's 16-row boxes are issued by as many lanes, each finding its
// box's block with one shuffle. A tile inside one block (block size a
// multiple of 64) is issued by lane 0 as one 64-row box per column half, as
// for the contiguous cache.
template <int D>
__device__ __forceinline__ void produce_paged(const DecodeParams& p, uint8_t* smem, StageInfo* info, uint64_t* full,
                                              uint64_t* empty, const CUtensorMap* tm_k64, const CUtensorMap* tm_v64,
                                              const CUtensorMap* tm_k16, const CUtensorMap* tm_v16, int lane) {
  using C = DecCfg<D>;
  constexpr unsigned kAll = 0xffffffffu;
  if (lane == 0) {
    prefetch_tensormap(tm_k64);
    prefetch_tensormap(tm_v64);
    prefetch_tensormap(tm_k16);
    prefetch_tensormap(tm_v16);
  }
  const uint64_t policy = l2_policy_evict_first();
  const int bs = p.block_size;
  const bool whole = bs % kDecTileKeys == 0;  // every full tile lies inside one block
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  int it = 0;  // ring position
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
    const ItemCoord c = item_coord(p, item);
    const int raw = __ldg(p.seqlens + c.b);
    const int len = valid_len(raw + p.len_add, p.S_max);
    if (lane == 0 && c.g == 0 && c.split == 0 && c.hsl == 0) {
      if (p.len_add ? (raw < 0 || raw >= p.S_max) : (len != raw))
        raise_error(p.len_add ? GQA_DEVERR_APPEND_POS : GQA_DEVERR_SEQLEN);
    }
    const int t_begin = c.split * p.chunk;
    const int t_end = min(len, t_begin + p.chunk);
    if (t_begin >= t_end) {
      if (c.split == 0) {  // an empty sequence: zeros for this item's heads
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)c.b * p.H + c.h0) * D);
        for (int i = lane; i < c.nh * D / 8; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      continue;
    }
    const int ntiles = (t_end - t_begin + kDecTileKeys - 1) / kDecTileKeys;
    const int32_t* trow = p.block_table + (size_t)c.b * p.max_blocks;
    const int blk_end = (t_end - 1) / bs + 1;  // the item's blocks: [t_begin / bs, blk_end)
    int win = t_begin / bs;                    // lane j holds the entry of block win + j
    int ent = win + lane < blk_end ? __ldg(trow + win + lane) : 0;
    for (int tt = 0; tt < ntiles && ok; ++tt, ++it) {
      const int s = it % C::kStages;
      const int t0 = t_begin + tt * kDecTileKeys;
      const int rows = min(kDecTileKeys, t_end - t0);
      const int last_blk = (t0 + rows - 1) / bs;
      if (last_blk >= win + 32) {  // the tile's blocks are past the window: the next 32
        win = t0 / bs;
        ent = win + lane < blk_end ? __ldg(trow + win + lane) : 0;
      }
      if (lane == 0 && it >= C::kStages) ok = mbar_wait_bounded(&empty[s], ((it / C::kStages) - 1) & 1);
      ok = __shfl_sync(kAll, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      uint8_t* stage = smem + s * C::kStageBytes;
      if (whole && rows == kDecTileKeys) {
        const int e = __shfl_sync(kAll, ent, t0 / bs - win);
        if (lane == 0) {
          const int new_row = (p.len_add && t0 <= len - 1 && len - 1 < t0 + rows) ? len - 1 - t0 : -1;
          info[s] = StageInfo{item, rows,
                              (tt == 0 ? kTileFirst : 0) | (tt == ntiles - 1 ? kTileLast : 0) |
                                  (len <= p.chunk ? kUnitSingleSplit : 0),
                              new_row};
          issue_tile<D>(stage, &full[s], tm_k64, tm_v64, tm_k16, tm_v16, paged_row(p, e, c.g, t0), rows, policy);
        }
      } else {
        // 16-row box bx (keys t0 + 16 bx ..) by lane bx; a box lies inside one block
        const int nbox = (rows + kDecBoxRows - 1) / kDecBoxRows;
        const int bx = lane < nbox ? lane : 0;
        const int e = __shfl_sync(kAll, ent, (t0 + bx * kDecBoxRows) / bs - win);
        if (lane == 0) {
          const int new_row = (p.len_add && t0 <= len - 1 && len - 1 < t0 + rows) ? len - 1 - t0 : -1;
          info[s] = StageInfo{item, rows,
                              (tt == 0 ? kTileFirst : 0) | (tt == ntiles - 1 ? kTileLast : 0) |
                                  (len <= p.chunk ? kUnitSingleSplit : 0),
                              new_row};
          mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * kDecBoxRows * 128 * C::kHalves * 2));
        }
        __syncwarp();
        if (lane < nbox) {
          const int brow = paged_row(p, e, c.g, t0 + bx * kDecBoxRows);
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf) {
            const int off = hf * C::kHalfBytes + bx * kDecBoxRows * 128;
            tma_load_2d(stage + off, tm_k16, hf * 64, brow, &full[s], policy);
            tma_load_2d(stage + C::kTileBytes + off, tm_v16, hf * 64, brow, &full[s], policy);
          }
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
      if (it >= C::kStages) ok = mbar_wait_bounded(&empty[s], ((it / C::kStages) - 1) & 1);
      if (ok) {
        info[s] = StageInfo{-1, 0, 0, 0};
        mbar_arrive(&full[s]);
        ++it;
      }
    }
    // this CTA's own loads must land before the block may exit
    for (int j = max(0, it - C::kStages); j < it; ++j) mbar_wait_bounded(&full[j % C::kStages], (j / C::kStages) & 1);
  }
}

// Keys of a CTA's first work item that it asks L2 for before its grid
// dependency resolves (K and V: 2 x 64 x 256 B = 32 KB per CTA for bf16
// d = 128), so that the DRAM reads of a decode call start while the kernel
// before it (the previous call's split combine, the tail of its decode)
// finishes.
#ifndef GQA_DEC_WARM_KEYS
#define GQA_DEC_WARM_KEYS 192
#endif
constexpr int kDecWarmKeys = GQA_DEC_WARM_KEYS;

// L2 warm-up of the first `max_keys` keys of work item `c` of a contiguous
// cache ([units * S_max] rows of kRowBytes): K and V rows from the item's
// first key, as far as the (possibly stale) length `raw` reaches. One head
// slice per unit asks; the others read the same rows.
template <int kRowBytes>
__device__ __forceinline__ void warm_first_item(const DecodeParams& p, const ItemCoord& c, int raw, int max_keys) {
  if (c.hsl != 0) return;
  const int len = valid_len(raw + p.len_add, p.S_max);
  const int t_begin = c.split * p.chunk;
  const int t_end = min(min(len, t_begin + p.chunk), t_begin + max_keys);
  if (t_end <= t_begin) return;
  const size_t off = ((size_t)c.unit * p.S_max + t_begin) * kRowBytes;
  const uint32_t bytes = (uint32_t)(t_end - t_begin) * kRowBytes;
  constexpr uint32_t kStep = 32768;  // bytes per prefetch instruction
  for (uint32_t o = 0; o < bytes; o += kStep) {
    const uint32_t n = min(kStep, bytes - o);
    prefetch_l2_bulk(static_cast<const uint8_t*>(p.k_cache_w) + off + o, n);
    prefetch_l2_bulk(static_cast<const uint8_t*>(p.v_cache_w) + off + o, n);
  }
}

// The paged form of warm_first_item, by the producer warp: lane i asks L2
// for the rows of block i of the item's first max_keys keys (a table entry
// read through L2 that may be stale; an entry outside the pool is skipped).
template <int D>
__device__ __forceinline__ void warm_first_item_paged(const DecodeParams& p, const ItemCoord& c, int raw, int max_keys,
                                                      int lane) {
  if (c.hsl != 0) return;
  const int len = valid_len(raw + p.len_add, p.S_max);
  const int t_begin = c.split * p.chunk;
  const int t_end = min(min(len, t_begin + p.chunk), t_begin + max_keys);
  if (t_end <= t_begin) return;
  const int bs = p.block_size;
  const int blk = t_begin / bs + lane;  // the lane's block of the sequence
  if (blk * bs >= t_end) return;
  const int e = __ldcg(p.block_table + (size_t)c.b * p.max_blocks + blk);
  if ((unsigned)e >= (unsigned)p.num_blocks) return;
  const int r0 = max(t_begin, blk * bs), r1 = min(t_end, (blk + 1) * bs);  // keys of the block to warm
  const size_t off = ((size_t)(e * p.K + c.g) * bs + (r0 - blk * bs)) * D * 2;
  const uint32_t bytes = (uint32_t)(r1 - r0) * D * 2;
  prefetch_l2_bulk(static_cast<const uint8_t*>(p.k_cache_w) + off, bytes);
  prefetch_l2_bulk(static_cast<const uint8_t*>(p.v_cache_w) + off, bytes);
}

// kPaged: the cache is a paged pool; kInt8: the cache holds 8-bit codes and
// per-row scales (tm_k*/tm_v* then map codes, tm_ks/tm_vs the scales; the
// bf16 kernels ignore tm_ks/tm_vs).
template <int D, bool kPaged, bool kInt8>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                       const DecodeParams p) {
  static_assert(!(kPaged && kInt8), "no paged 8-bit cache");
  using C = DecCfg<D, kInt8>;
  extern __shared__ __align__(1024) uint8_t smem[];
  float* merge = reinterpret_cast<float*>(smem + C::kMergeOff);
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + C::kInfoOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kStages;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (smem_u32(smem) & 1023u) {  // the swizzle pattern needs 1024-byte aligned stages
    grid_dep_wait();
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  // Launched as a programmatic dependent: until grid_dep_wait() returns, the
  // previous kernel on the stream may still be running. Before it: the
  // barriers, the descriptor prefetch, and an L2 warm-up of the first work
  // item's key rows (of a paged cache through its table), sized by a length
  // read that may be stale -- a hint only, so the rows may still be being
  // written. After it the length is read again and every input is read for
  // real.
  int spec_first = 0;
  if (!kPaged && warp == kDecConsumerWarps && lane == 0) {
    prefetch_tensormap(&tm_k64);
    prefetch_tensormap(&tm_v64);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    if constexpr (kInt8) {
      prefetch_tensormap(&tm_ks);
      prefetch_tensormap(&tm_vs);
    }
    // through L2 only (ld.cg): no L1 line of the possibly stale value survives the wait
    if ((int)blockIdx.x < p.nitems) spec_first = __ldcg(p.seqlens + item_coord(p, blockIdx.x).b);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (!kPaged && warp == kDecConsumerWarps && lane == 0 && (int)blockIdx.x < p.nitems)
    warm_first_item<D * C::kElt>(p, item_coord(p, blockIdx.x), spec_first, kDecWarmKeys);
  if (kPaged && warp == kDecConsumerWarps && (int)blockIdx.x < p.nitems) {
    const ItemCoord c0 = item_coord(p, blockIdx.x);
    warm_first_item_paged<D>(p, c0, __ldcg(p.seqlens + c0.b), kDecWarmKeys, lane);
  }
  grid_dep_wait();
  // the combine kernel (or the next decode) may be scheduled now; it waits for this grid to finish
  grid_dep_launch();

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if constexpr (kPaged) {
      produce_paged<D>(p, smem, info, full, empty, &tm_k64, &tm_v64, &tm_k, &tm_v, lane);
    } else if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      int it = 0;  // ring position
      bool ok = true;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      for (int k = 0;; ++k) {
        // the first item of each CTA is its block index; later ones come from the counter
        const int ticket = k == 0 ? 1 : take_ticket(p.ws_queue, p.tag);
        const int item = k == 0 ? (int)blockIdx.x : (int)gridDim.x + ticket - 1;
        if (ticket <= 0 || item >= p.nitems) break;
        const ItemCoord c = item_coord(p, item);
        const int raw = __ldg(p.seqlens + c.b);
        const int len = valid_len(raw + p.len_add, p.S_max);
        if (c.g == 0 && c.split == 0 && c.hsl == 0) {
          if (p.len_add ? (raw < 0 || raw >= p.S_max) : (len != raw)) {
            raise_error(p.len_add ? GQA_DEVERR_APPEND_POS : GQA_DEVERR_SEQLEN);
          }
        }
        const int t_begin = c.split * p.chunk;
        const int t_end = min(len, t_begin + p.chunk);
        if (t_begin >= t_end) {
          if (c.split == 0) {  // an empty sequence: zeros for this item's heads
            uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)c.b * p.H + c.h0) * D);
            for (int i = 0; i < c.nh * D / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
          }
          continue;
        }
        const int ntiles = (t_end - t_begin + kDecTileKeys - 1) / kDecTileKeys;
        for (int tt = 0; tt < ntiles && ok; ++tt, ++it) {
          const int s = it % C::kStages;
          const int t0 = t_begin + tt * kDecTileKeys;
          const int rows = min(kDecTileKeys, t_end - t0);
          if (it >= C::kStages) ok = mbar_wait_bounded(&empty[s], ((it / C::kStages) - 1) & 1);
          if (!ok) break;
#ifdef GQA_WAIT_TEST
          // The wait-test build of the library (never the product): the first
          // CTA issues nothing for its first item's second tile, so the stage's
          // full barrier never completes and the consumers' bounded wait on it
          // runs out. No load is in flight for that stage when they give up.
          if (blockIdx.x == 0 && k == 0 && tt == 1) continue;
#endif
          const int new_row = (p.len_add && t0 <= len - 1 && len - 1 < t0 + rows) ? len - 1 - t0 : -1;
          info[s] = StageInfo{item, rows,
                              (tt == 0 ? kTileFirst : 0) | (tt == ntiles - 1 ? kTileLast : 0) |
                                  (len <= p.chunk ? kUnitSingleSplit : 0),
                              new_row};
          if constexpr (kInt8)
            issue_tile_i8<D>(smem + s * C::kStageBytes, &full[s], &tm_k64, &tm_v64, &tm_k, &tm_v, &tm_ks, &tm_vs,
                             c.unit * p.S_max + t0, c.unit, t0, rows,
                             static_cast<const __nv_bfloat16*>(p.q) + ((size_t)c.b * p.H + c.h0) * D,
                             tt == 0 ? (uint32_t)(c.nh * D * 2) : 0u, policy);
          else
            issue_tile<D>(smem + s * C::kStageBytes, &full[s], &tm_k64, &tm_v64, &tm_k, &tm_v, c.unit * p.S_max + t0,
                          rows, policy);
        }
        if (!ok) break;
      }
      leave_queue(p.ws_queue, p.tag);
      // no more work: a record without loads ends the consumers' loop
      if (ok) {
        const int s = it % C::kStages;
        if (it >= C::kStages) ok = mbar_wait_bounded(&empty[s], ((it / C::kStages) - 1) & 1);
        if (ok) {
          info[s] = StageInfo{-1, 0, 0, 0};
          mbar_arrive(&full[s]);
          ++it;
        }
      }
      // this CTA's own loads must land before the block may exit
      for (int j = max(0, it - C::kStages); j < it; ++j) mbar_wait_bounded(&full[j % C::kStages], (j / C::kStages) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;  // 0..127
  const int kb = warp * 16;
  uint32_t qf[D / 16][2];
  float qb_a = 0.f, qb_b = 0.f;  // 8-bit path: the code bias of the scores
  int ti = 0;                    // 8-bit path: index of the tile in its work item
  WarpState<D> st;
  ItemCoord cur{};
  for (int it = 0;; ++it) {
    const int s = it % C::kStages;
    if (!mbar_wait_bounded(&full[s], (it / C::kStages) & 1)) break;  // every consumer warp sees the same barrier
    const StageInfo si = info[s];
    if (si.item < 0) break;
    if (si.flags & kTileFirst) {
      cur = item_coord(p, si.item);
      const __nv_bfloat16* qh = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)cur.b * p.H + cur.h0) * D;
      if constexpr (kInt8) {  // the producer brought the item's q rows with its first tile
        load_q_frag_i8<D>(qf, reinterpret_cast<const __nv_bfloat16*>(smem + s * C::kStageBytes + C::kQOff), lane,
                          cur.nh);
        q_code_bias<D>(qf, lane, qb_a, qb_b);
        ti = 0;
      } else
        load_q_frag<D>(qf, qh, lane, cur.nh);
      st.reset();
    }
    if constexpr (!kInt8) {  // the fused append (bf16 caches only)
      if (si.new_row >= 0 && (si.new_row >> 4) == warp)
        append_row<D, kPaged>(p, cur, smem + s * C::kStageBytes, si.new_row, lane);
    }
    if constexpr (kInt8) {
      // warps 0-1 take the even tiles of a work item and warps 2-3 the odd
      // ones, 32 keys each, so that a warp has two tile times for every tile
      // it computes; the last tile of an odd count goes to all four warps,
      // 16 keys each. Which warp sums which keys follows from the item alone,
      // not from the order in which CTAs take items.
      const float* sk = reinterpret_cast<const float*>(smem + s * C::kStageBytes + C::kScaleOff);
      const uint32_t sa = smem_u32(smem + s * C::kStageBytes);
      if ((si.flags & kTileLast) && (ti & 1) == 0) {
        if (kb < si.rows)
          warp_tile_i8<D, 1>(st, qf, qb_a, qb_b, sa, sk, sk + kDecTileKeys, kb, si.rows, lane, p.scale_log2);
      } else if ((ti & 1) == (warp >> 1)) {
        const int kb8 = (warp & 1) * 32;
        if (kb8 < si.rows)
          warp_tile_i8<D, 2>(st, qf, qb_a, qb_b, sa, sk, sk + kDecTileKeys, kb8, si.rows, lane, p.scale_log2);
      }
      ++ti;
    } else if (kb < si.rows) {
      warp_tile<D>(st, qf, smem_u32(smem + s * C::kStageBytes), kb, si.rows, lane, p.scale_log2);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (si.flags & kTileLast)
      item_epilogue<D, kInt8>(p, cur, st, merge, (si.flags & kUnitSingleSplit) != 0, tid, warp, lane);
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
// Split-KV combine (the log-sum-exp merge of the partials):
//   M = max_s m_s,  out[b,h] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// over the ns = ceil(len_b / chunk) splits that hold keys (units with one
// split were finished by the decode kernel). CS CTAs per (b, h), each for
// D / CS columns; in a CTA of NT threads, RL = D / (4 CS) threads cover one
// partial row (a 16-byte column group each) and the NT / RL row slots take
// every (NT / RL)-th split, kBatch rows each loaded before anything waits.
// Launched as a programmatic dependent of the decode kernel: the length is
// read before the grid dependency (the decode kernel does not write it), the
// partials after it.
template <int D, int NT, int CS>
struct CombineCfg {
  static constexpr int RL = D / 4 / CS;  // threads per partial row
  static constexpr int R = NT / RL;      // row slots
  static constexpr int kBatch = (160 + R - 1) / R < 8 ? (160 + R - 1) / R : 8;  // up to 160 rows in the first round
  static_assert(RL >= 1 && RL <= 32 && NT % RL == 0 && NT % 32 == 0, "combine shape");
};

template <typename OutT, int D, int NT, int CS>
__global__ void __launch_bounds__(NT) decode_combine_kernel(OutT* __restrict__ out, const float* __restrict__ ws_o,
                                                            const float2* __restrict__ ws_ml,
                                                            const int32_t* __restrict__ seqlens, int len_add, int H,
                                                            int K, int S_max, int G, int chunk, int nsplit,
                                                            int skip_single) {
  using CC = CombineCfg<D, NT, CS>;
  constexpr int RL = CC::RL, R = CC::R, kBatch = CC::kBatch, NW = NT / 32;
  __shared__ float sw[kMaxCombineSplits];
  __shared__ float4 sacc[R][RL];
  __shared__ float sred[2 * NW];
  const int bh = blockIdx.x / CS, slice = blockIdx.x % CS;
  const int b = bh / H, h = bh % H;
  const int g = h / G, j = h % G;
  const int len = valid_len(__ldg(seqlens + b) + len_add, S_max);
  const int ns = (len + chunk - 1) / chunk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = tid % RL, slot = tid / RL;
  OutT* orow = out + (size_t)bh * D + slice * (D / CS);
  // The next kernel on the stream (the next decode call) may be scheduled now:
  // it only warms L2 until its own grid dependency, which includes this grid.
  grid_dep_launch();
  grid_dep_wait();
  if (ns == 0) {  // empty sequence
    for (int i = tid; i < D / CS; i += NT) store_out<OutT>(orow + i, 0.f);
    return;
  }
  if (ns == 1 && skip_single) return;
  const size_t base = ((size_t)(b * K + g) * nsplit) * G + j;  // split s at base + s*G
  const float* obase = ws_o + base * D + slice * (D / CS);
  // every load of the first round goes out before anything waits on one
  float2 ml = tid < ns ? __ldcg(&ws_ml[base + (size_t)tid * G]) : make_float2(-INFINITY, 0.f);
  float4 v[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int sp = slot + R * u;
    v[u] = sp < ns ? __ldcg(reinterpret_cast<const float4*>(obase + (size_t)sp * G * D) + col)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // M = max m_s
  float M = ml.x;
  for (int sp = tid + NT; sp < ns; sp += NT) M = fmaxf(M, __ldcg(&ws_ml[base + (size_t)sp * G].x));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) sred[warp] = M;
  __syncthreads();
  M = sred[0];
#pragma unroll
  for (int q = 1; q < NW; ++q) M = fmaxf(M, sred[q]);
  // weights 2^(m_s - M) and L = sum l_s 2^(m_s - M)
  float L = 0.f;
  if (tid < ns) {
    const float f = fast_exp2(ml.x - M);
    sw[tid] = f;
    L = ml.y * f;
  }
  for (int sp = tid + NT; sp < ns; sp += NT) {
    const float2 m2 = __ldcg(&ws_ml[base + (size_t)sp * G]);
    const float f = fast_exp2(m2.x - M);
    sw[sp] = f;
    L += m2.y * f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  if (lane == 0) sred[NW + warp] = L;
  __syncthreads();
  // weighted sum of the partial O rows: the loaded batch, then any further splits
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int sp = slot + R * u;
    const float f = sp < ns ? sw[sp] : 0.f;
    acc.x += v[u].x * f;
    acc.y += v[u].y * f;
    acc.z += v[u].z * f;
    acc.w += v[u].w * f;
  }
  for (int s0 = slot + R * kBatch; s0 < ns; s0 += R * kBatch) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int sp = s0 + R * u;
      v[u] = sp < ns ? __ldcg(reinterpret_cast<const float4*>(obase + (size_t)sp * G * D) + col)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int sp = s0 + R * u;
      const float f = sp < ns ? sw[sp] : 0.f;
      acc.x += v[u].x * f;
      acc.y += v[u].y * f;
      acc.z += v[u].z * f;
      acc.w += v[u].w * f;
    }
  }
  sacc[slot][col] = acc;
  __syncthreads();
  if (tid < RL) {
    float Lt = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) Lt += sred[NW + q];
    const float inv = 1.f / Lt;
    float4 t = sacc[0][tid];
#pragma unroll 8
    for (int q = 1; q < R; ++q) {
      t.x += sacc[q][tid].x;
      t.y += sacc[q][tid].y;
      t.z += sacc[q][tid].z;
      t.w += sacc[q][tid].w;
    }
    OutT* o = orow + tid * 4;
    store_out<OutT>(o + 0, t.x * inv);
    store_out<OutT>(o + 1, t.y * inv);
    store_out<OutT>(o + 2, t.z * inv);
    store_out<OutT>(o + 3, t.w * inv);
  }
}

}  // namespace gqa
