// Causal GQA prefill, two heads of one KV group per work unit, on the
// 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   out[b, i, h, :] = sum_{j <= i} softmax_j(scale * q[b,i,h] . k[b,j,g]) v[b,j,g],  g = h / (H/K)
//
// A work unit is one 128-row query tile of two query heads h0 = g G + 2 p and
// h0 + 1 of KV group g (G even): the two tiles need exactly the same K/V
// tiles and the same causal extent, so every K/V tile the CTA loads serves
// both ("GQA 完全拆解", section 工程实现: the group's query heads share one
// load of each KV block). Persistent CTAs, one per SM, take units from a
// list ordered heaviest first (see cta_unit).
//
// Warp roles (18 warps):
//   warps 8 t + 4 h + q (t, h in {0, 1}, q = 0..3): the softmax of tile t
//              for keys 64 h .. 64 h + 63 of each 128-key tile; thread q 32 +
//              lane owns query row q 32 + lane (TMEM lane). The two warps
//              with the same t and q hold the same rows (partner warps) and
//              exchange row maxima, checks and sums through shared memory,
//              each exchange closed by an mbarrier of 64 arrivals (one per
//              pair of warps and tile; its wait is bounded like the others).
//   warp 16    TMEM allocation; the converged warp issues every tcgen05.mma
//              from one elected lane
//   warp 17    TMA loads: lane 0 the K tiles, lane 1 the V tiles, lane 2 the
//              Q tiles (128 keys per K/V tile, two stages each); the owner of
//              a key tile also stores it to the KV cache from shared memory
// TMEM (512 columns): S_t at columns 128 t (fp32, 128 keys) and O_t at
// 256 + 128 t (fp32, D columns). Each softmax half writes its P (bf16 pairs)
// over the first 32 of its own 64 score columns, and P_t V is issued with A
// read from TMEM, so P never goes through shared memory.
//
// The chain of a tile from one softmax step to the next is kept short:
//   * P_t(j) V is issued in two halves, each as soon as the softmax warps
//     of that key half have stored their P;
//   * S_t(j+1) follows the second half (it overwrites P_t(j)), and its
//     completion hands it to the softmax;
//   * the softmax computes the exponentials against the running maximum
//     without a pass over the row for a new one: the sum of a tile's P is at
//     most 2^8 unless some P exceeds 2^8, and only then (rare after a row's
//     first tile) is the row maximum taken and the tile recomputed from S,
//     still intact in TMEM. So P stays at most 2^8, and O_t is rescaled only
//     when a row's maximum grows by more than 2^8.
// The two tiles take turns, so the tensor pipe has the other tile's work
// while a softmax runs. Operations issued by one thread complete in order,
// so S_t(j+1) runs after the P V that reads P_t(j), and the commit after it
// covers every MMA before it: a softmax thread that sees S_t(j+1) may
// rescale O_t.
#pragma once

#include <atomic>

#include "common.cuh"
#include "prefill.cuh"
#include "tcgen05.cuh"

namespace gqa {

constexpr int kPpBM = 128;      // query rows per tile
constexpr int kPpBN = 128;      // keys per K/V tile and per S tile
constexpr int kPpStages = 2;    // K and V ring stages
constexpr int kPpThreads = 576;
constexpr int kPpTmemCols = 512;
constexpr int kPpMmaWarp = 16;
// Every kPpPolyEvery-th pair of exponentials is computed on the FMA pipe
// (exp2_poly2), the rest by the MUFU unit; 0: all by the MUFU unit. One in
// eight measured fastest (0.527 ms against 0.538 with none and 0.556 with one
// in four on the 4 x 4096 x 32 x 128 prefill).
#ifndef GQA_PP_POLY_EVERY
#define GQA_PP_POLY_EVERY 8
#endif
constexpr int kPpPolyEvery = GQA_PP_POLY_EVERY;
__device__ __forceinline__ bool pp_wait(uint64_t* bar, uint32_t parity) { return mbar_wait_bounded(bar, parity); }
constexpr int kPpLoadWarp = 17;
constexpr int kPpMaxSeqs = 256;  // prompts of a packed batch that the unit list takes (8 per lane)
constexpr int kPpListMax = 512;  // units per CTA that the unit list holds

template <int D>
struct PpCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kQHalf = kPpBM * 128;      // one 64-column half of a Q tile
  static constexpr int kKVHalf = kPpBN * 128;     // one 64-column half of a K or V tile
  static constexpr int kQBytes = kHalves * kQHalf;
  static constexpr int kKVBytes = kHalves * kKVHalf;
  static constexpr int kQOff = 0;                                 // Q0, Q1
  static constexpr int kKOff = kQOff + 2 * kQBytes;               // K stages
  static constexpr int kVOff = kKOff + kPpStages * kKVBytes;      // V stages
  static constexpr int kXOff = kVOff + kPpStages * kKVBytes;  // partner exchange [2 tiles][2 slots][2 halves][128]
  static constexpr int kBarOff = kXOff + 2 * 2 * 2 * kPpBM * 4;
  // q_full[2] q_empty[2] k_full[S] k_empty[S] v_full[S] v_empty[S] s_full[2] p_lo[2] p_hi[2] o_ready[2]
  // o_free[2] mma_done pair[8]
  static constexpr int kNumBars = 4 + 4 * kPpStages + 10 + 1 + 8;
  // packed batches: this CTA's unit list [kPpListMax] (uint2) and its length
  static constexpr int kListOff = (kBarOff + kNumBars * 8 + 16 + 15) / 16 * 16;
  static constexpr int kListCountOff = kListOff + kPpListMax * 8;
  static constexpr int kSmemBytes = kListCountOff + 16;
  static constexpr int kOCol = 256;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct PairParams {
  void* out;                  // [B, S, H, D] bf16, or packed [T, H, D]
  void* k_cache;              // [B, K, S_max, D] bf16, or null: no cache write
  void* v_cache;
  const int32_t* cu_seqlens;  // varlen: [B + 1]; null: fixed length S
  int B, S, H, K, G, S_max, T;
  int ordered;                // varlen: units from the per-CTA list (build_unit_list); 0: sequence-major
  float scale_log2;
};

// The work list, heaviest units first (a unit's cost is its qt + 1 key
// tiles), and which entries a CTA takes.
//   Prompts of one length: level r holds query tile nqt - 1 - r of every
// sequence, sequence by sequence, then groups, then the head pairs of a group
// (the two pairs of a group read the same K/V tiles at about the same time).
// CTA c takes the entries k * grid + c for even k and k * grid + grid - 1 - c
// for odd k, a snake over the levels, so every CTA gets the same mix of heavy
// and light units. Counted in key tiles, taking every grid-th entry of a
// sequence-major list left the busiest CTA 12 % above the mean on 4 x 4096
// tokens, the snake 0.3 %; measured, the call is 3 % faster (the SMs that
// finish early let the others run at a higher clock under the power cap).
//   Packed batches of at most kPpMaxSeqs prompts: the same level order and
// snake, a level now being a query tile index (build_unit_list), so a level
// holds the units of equal cost of every prompt long enough to have one.
// Counted in key tiles plus a per-unit cost, the busiest CTA of 8 prompts of
// 915-3749 tokens is 1 % above the mean this way, against 8 % for every
// grid-th entry of a sequence-major list and 20 % for levels counted down
// from each prompt's own last tile; measured, the call is 6.5 % faster than
// with the sequence-major list. Larger batches, and CTA shares beyond the
// list: sequence by sequence, each sequence's heaviest query tiles first, CTA
// c taking every grid-th entry from c.
__device__ __forceinline__ int cta_unit(const PairParams& p, int k) {
  const bool snake = p.cu_seqlens == nullptr && (k & 1);
  return k * (int)gridDim.x + (snake ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
}

// List entry u -> sequence b (rows seq0 .. seq0 + len - 1), query tile qt,
// group g, head pair pr. Returns false past the last unit.
__device__ __forceinline__ bool pair_unit(const PairParams& p, int u, int& b, int& seq0, int& len, int& qt, int& g,
                                          int& pr) {
  const int per_qt = p.K * (p.G / 2);
  if (p.cu_seqlens == nullptr) {
    const int nqt = (p.S + kPpBM - 1) / kPpBM;
    const int per_lvl = p.B * per_qt;
    const int r = u / per_lvl;
    if (r >= nqt) return false;
    const int rem = u % per_lvl;
    b = rem / per_qt;
    qt = nqt - 1 - r;
    g = (rem % per_qt) / (p.G / 2);
    pr = rem % (p.G / 2);
    seq0 = b * p.S;
    len = p.S;
    return true;
  }
  int acc = 0;
  for (int bb = 0; bb < p.B; ++bb) {
    int s0 = __ldg(p.cu_seqlens + bb), s1 = __ldg(p.cu_seqlens + bb + 1);
    s0 = min(max(s0, 0), p.T);  // clamped to the packed rows (bad offsets are reported once, by the kernel)
    s1 = min(max(s1, s0), p.T);
    const int n = (s1 - s0 + kPpBM - 1) / kPpBM * per_qt;
    if (u < acc + n) {
      const int r = u - acc;
      b = bb;
      seq0 = s0;
      len = s1 - s0;
      qt = (len + kPpBM - 1) / kPpBM - 1 - r / per_qt;
      g = (r % per_qt) / (p.G / 2);
      pr = r % (p.G / 2);
      return true;
    }
    acc += n;
  }
  return false;
}

// Packed batches of at most kPpMaxSeqs prompts (p.ordered): the list in the
// order of the fixed-length case -- level by level, a level being a query
// tile index qt from the highest down (its units cost qt + 1 key tiles each),
// within a level the prompts that have a tile qt in order, then groups, then
// head pairs -- and the same snake over the CTAs. Warp-collective, run by
// one warp before the roles start: writes this CTA's entries (prompt |
// head-pair index << 8, qt) and their count to shared memory. The work is one
// pass over the levels with a ballot per 32 prompts, then a few instructions
// per entry. The host takes this form only when every CTA's share fits the
// list.
template <int D>
__device__ __forceinline__ void build_unit_list(const PairParams& p, uint8_t* smem, int lane) {
  using C = PpCfg<D>;
  constexpr int kChunks = kPpMaxSeqs / 32;
  int nq[kChunks];  // query tiles of prompt 32 j + lane
  int top = 0;
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    const int bb = 32 * j + lane;
    nq[j] = 0;
    if (bb < p.B) {
      int s0 = __ldg(p.cu_seqlens + bb), s1 = __ldg(p.cu_seqlens + bb + 1);
      s0 = min(max(s0, 0), p.T);  // clamped as in pair_unit
      s1 = min(max(s1, s0), p.T);
      nq[j] = (s1 - s0 + kPpBM - 1) / kPpBM;
    }
    top = max(top, nq[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = max(top, __shfl_xor_sync(0xffffffffu, top, o));
  const int per_qt = p.K * (p.G / 2);
  const int c = (int)blockIdx.x, grid = (int)gridDim.x;
  uint2* list = reinterpret_cast<uint2*>(smem + C::kListOff);
  int n = 0;      // entries written
  int u = c;      // list position of entry n: n grid + c for even n, n grid + grid - 1 - c for odd n
  int above = 0;  // units in the levels above qt
  for (int qt = top - 1; qt >= 0 && n < kPpListMax; --qt) {
    unsigned m[kChunks];  // prompts with a query tile qt
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      m[j] = __ballot_sync(0xffffffffu, nq[j] > qt);
      cnt += __popc(m[j]);
    }
    const int end = above + cnt * per_qt;
    while (u < end && n < kPpListMax) {
      const int r = u - above;
      int i = r / per_qt, b = -1;  // b: the i-th prompt with a tile qt
#pragma unroll
      for (int j = 0; j < kChunks; ++j) {
        const int pc = __popc(m[j]);
        if (b < 0) {
          if (i < pc) {
            unsigned mm = m[j];
            for (int t = 0; t < i; ++t) mm &= mm - 1u;
            b = 32 * j + __ffs((int)mm) - 1;
          } else {
            i -= pc;
          }
        }
      }
      if (lane == 0) list[n] = make_uint2((unsigned)b | ((unsigned)(r % per_qt) << 8), (unsigned)qt);
      ++n;
      u = n * grid + ((n & 1) ? grid - 1 - c : c);
    }
    above = end;
  }
  if (lane == 0) *reinterpret_cast<int*>(smem + C::kListCountOff) = n;
}

// Unit k of this CTA: from the list for packed batches that have one, else
// entry cta_unit(k) of the list that pair_unit decodes.
template <int D>
__device__ __forceinline__ bool pp_unit(const PairParams& p, const uint8_t* smem, int k, int& b, int& seq0, int& len,
                                        int& qt, int& g, int& pr) {
  using C = PpCfg<D>;
  if (p.ordered) {
    if (k >= *reinterpret_cast<const int*>(smem + C::kListCountOff)) return false;
    const uint2 e = reinterpret_cast<const uint2*>(smem + C::kListOff)[k];
    b = (int)(e.x & 0xffu);
    const int rem = (int)(e.x >> 8);
    qt = (int)e.y;
    g = rem / (p.G / 2);
    pr = rem % (p.G / 2);
    int s0 = __ldg(p.cu_seqlens + b), s1 = __ldg(p.cu_seqlens + b + 1);
    s0 = min(max(s0, 0), p.T);
    s1 = min(max(s1, s0), p.T);
    seq0 = s0;
    len = s1 - s0;
    return true;
  }
  return pair_unit(p, cta_unit(p, k), b, seq0, len, qt, g, pr);
}

// The key tile j of unit (b, g, len) to the cache, from its copy in shared
// memory (a K or V tile of 128 rows, 64-column halves, 128-byte swizzle):
// full tiles and whole 16-row groups by TMA store, the last rows of a
// partial group by plain stores. Only rows below min(len, S_max) are written.
// Called by the one thread that loaded the tile, after the tile landed; it
// waits for the stores to have read shared memory before returning.
template <int D>
__device__ __forceinline__ void store_tile_to_cache(const PairParams& p, const uint8_t* tile, const CUtensorMap* tm_full,
                                                    const CUtensorMap* tm16, void* cache, int b, int g, int len,
                                                    int j) {
  using C = PpCfg<D>;
  const int t0 = j * kPpBN;
  const int rows = min(min(len, p.S_max) - t0, kPpBN);
  if (rows <= 0) return;
  const int slab_row = (b * p.K + g) * p.S_max + t0;  // cache row of key t0
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (rows == kPpBN) {
#pragma unroll
    for (int hf = 0; hf < C::kHalves; ++hf)
      asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                       reinterpret_cast<uint64_t>(tm_full)),
                   "r"(hf * 64), "r"(slab_row), "r"(smem_u32(tile + hf * C::kKVHalf))
                   : "memory");
  } else {
    const int groups = rows / 16;
    for (int gi = 0; gi < groups; ++gi)
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                         reinterpret_cast<uint64_t>(tm16)),
                     "r"(hf * 64), "r"(slab_row + gi * 16), "r"(smem_u32(tile + hf * C::kKVHalf + gi * 2048))
                     : "memory");
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(cache);
    for (int r = groups * 16; r < rows; ++r)
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(tile + hf * C::kKVHalf + sw128((uint32_t)r, (uint32_t)ch));
          reinterpret_cast<uint4*>(dst + ((size_t)slab_row + r) * D + hf * 64)[ch] = v;
        }
  }
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// 16 TMEM columns of this thread's lane from 16 registers of bf16 pairs
__device__ __forceinline__ void tmem_st16_u(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M = 128 rows in lanes 0-127, 16
// bf16 of K in 8 columns, two per column, the lower k in the low half)
__device__ __forceinline__ void tc_mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// (d0, d1) = (a0, a1) * (b0, b1) + (c, c), each lane rounded once
__device__ __forceinline__ void fma2v(float& d0, float& d1, float a0, float a1, float b0, float b1, float c) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %6};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c));
}

// (d0, d1) = (a0, a1) + (b0, b1)
__device__ __forceinline__ void add2v(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 2^y0, 2^y1 for y <= 8 (y may be -inf) on the FMA pipe, for a share of the
// softmax's exponentials so that the MUFU unit (16 per clock per SM, as many
// exponentials per 128 x 128 tile as the tensor cores take clocks for its
// two products at d = 128) does not set the pace. y = r + f with r =
// round(y): adding 1.5 * 2^23 leaves r in the low mantissa bits of t, and
// f = y - r lies in [-0.5, 0.5]. 2^f is a cubic whose coefficients were
// fitted here by least squares on the relative error over [-0.5, 0.5]
// (largest relative error 7.5e-5 evaluated in float32, far below bf16's
// 2^-9). 2^r is applied by adding r << 23 to the exponent field, and
// bits(t) << 23 is exactly that: the bits of 1.5 * 2^23 shift out. y < -125
// (a masked score) gives 0.
__device__ __forceinline__ void exp2_poly2(float y0, float y1, float& e0, float& e1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  const float a0 = fmaxf(y0, -125.f), a1 = fmaxf(y1, -125.f);
  float t0, t1, r0, r1, f0, f1, p0, p1;
  add2v(t0, t1, a0, a1, kRound, kRound);
  add2v(r0, r1, t0, t1, -kRound, -kRound);
  add2v(f0, f1, a0, a1, -r0, -r1);
  fma2(p0, p1, f0, f1, 0.0551704988f, 0.242608517f);
  fma2v(p0, p1, p0, p1, f0, f1, 0.693260968f);
  fma2v(p0, p1, p0, p1, f0, f1, 0.999928236f);
  e0 = y0 < -125.f ? 0.f : __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = y1 < -125.f ? 0.f : __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

template <int D>
__global__ void __launch_bounds__(kPpThreads, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc128,
                        const __grid_constant__ CUtensorMap tm_vc128, const __grid_constant__ CUtensorMap tm_kc16,
                        const __grid_constant__ CUtensorMap tm_vc16, const PairParams p) {
  using C = PpCfg<D>;
  constexpr int S = kPpStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;              // [2 tiles] Q_t landed
  uint64_t* q_empty = bars + 2;         // [2 tiles] the unit's last S_t finished (Q_t may be replaced)
  uint64_t* k_full = bars + 4;          // [S stages]
  uint64_t* k_empty = k_full + S;       // [S] every S of the tile finished
  uint64_t* v_full = k_empty + S;
  uint64_t* v_empty = v_full + S;       // both P V of the tile finished
  uint64_t* s_full = v_empty + S;       // [2 tiles] S_t complete (and every MMA before it)
  uint64_t* p_lo = s_full + 2;          // [2 tiles] P_t of keys 0-63 stored (O_t rescaled): 128 arrivals
  uint64_t* p_hi = p_lo + 2;            // [2 tiles] P_t of keys 64-127 stored: 128 arrivals
  uint64_t* o_ready = p_hi + 2;         // [2 tiles] the unit's last P_t V finished
  uint64_t* o_free = o_ready + 2;       // [2 tiles] the epilogue has read O_t: 256 arrivals
  uint64_t* mma_done = o_free + 2;      // every MMA of the CTA finished (before TMEM is released)
  uint64_t* pair = mma_done + 1;        // [2 tiles][4 row groups] the partner warps' exchanges: 64 arrivals
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (smem_u32(smem) & 1023u) {  // the 128-byte swizzle assumes 1024-byte aligned tiles
    if (threadIdx.x == 0) raise_error(GQA_DEVERR_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_lo[i], 128);
      mbar_init(&p_hi[i], 128);
      mbar_init(&o_ready[i], 1);
      mbar_init(&o_free[i], 256);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&pair[i], 64);
    fence_mbar_init();
  }
  if (warp == kPpMmaWarp) {
    tmem_alloc(tmem_holder, kPpTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (p.ordered) {
    if (warp == 0) build_unit_list<D>(p, smem, lane);
    __syncthreads();
  }
  if (p.cu_seqlens && blockIdx.x == 0 && threadIdx.x == 0) {  // offsets outside the packed rows
    for (int bb = 0; bb < p.B; ++bb) {
      const int s0 = __ldg(p.cu_seqlens + bb), s1 = __ldg(p.cu_seqlens + bb + 1);
      if (s0 < 0 || s1 > p.T || s1 < s0) {
        raise_error(GQA_DEVERR_SEQLEN);
        break;
      }
    }
  }

  if (warp == kPpLoadWarp) {
    // ------------------------------------------------------------- loads
    if (lane < 3) {
      const int role = lane;  // 0: K tiles, 1: V tiles, 2: Q tiles
      const CUtensorMap* tm = role == 0 ? &tm_k : role == 1 ? &tm_v : &tm_q;
      prefetch_tensormap(tm);
      const uint64_t pol = role == 2 ? l2_policy_evict_first() : l2_policy_evict_last();
      uint64_t* full = role == 0 ? k_full : v_full;
      uint64_t* empty = role == 0 ? k_empty : v_empty;
      const int off = role == 0 ? C::kKOff : C::kVOff;
      int n = 0;  // tiles (or units, for Q) issued
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int b, seq0, len, qt, g, pr;
        if (!pp_unit<D>(p, smem, k, b, seq0, len, qt, g, pr)) break;
        if (role == 2) {
          for (int t = 0; t < 2 && ok; ++t) {
            if (n >= 1 && !(ok = pp_wait(&q_empty[t], (n - 1) & 1))) break;
            mbar_arrive_expect_tx(&q_full[t], C::kQBytes);
#pragma unroll
            for (int hf = 0; hf < C::kHalves; ++hf)
              tma_load_3d(smem + C::kQOff + t * C::kQBytes + hf * C::kQHalf, &tm_q, hf * 64, g * p.G + 2 * pr + t,
                          seq0 + qt * kPpBM, &q_full[t], pol);
          }
          ++n;
          continue;
        }
        const bool owner = p.k_cache != nullptr && pr == 0;  // writes its diagonal key tile qt
        for (int j = 0; j <= qt && ok; ++j, ++n) {
          const int s = n % S;
          if (n >= S && !(ok = pp_wait(&empty[s], ((n / S) - 1) & 1))) break;
          uint8_t* dst = smem + off + s * C::kKVBytes;
          mbar_arrive_expect_tx(&full[s], C::kKVBytes);
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d(dst + hf * C::kKVHalf, tm, hf * 64, g, seq0 + j * kPpBN, &full[s], pol);
          if (owner && j == qt) {
            if (!(ok = pp_wait(&full[s], (n / S) & 1))) break;
            store_tile_to_cache<D>(p, dst, role == 0 ? &tm_kc128 : &tm_vc128, role == 0 ? &tm_kc16 : &tm_vc16,
                                   role == 0 ? p.k_cache : p.v_cache, b, g, len, j);
          }
        }
      }
      // this CTA's loads land before it may exit
      if (role == 2) {
        for (int t = 0; t < 2; ++t)
          if (n >= 1) pp_wait(&q_full[t], (n - 1) & 1);
      } else {
        for (int i = max(0, n - S); i < n; ++i) pp_wait(&full[i % S], (i / S) & 1);
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // the cache stores are complete
      }
    }
  } else if (warp == kPpMmaWarp) {
    // --------------------------------------------------------------- MMA
    // The whole warp runs this loop converged, so descriptors and TMEM
    // addresses are warp-uniform values; one elected lane issues each
    // tcgen05.mma and commit. (Issued from a divergent single-lane branch,
    // every MMA paid for moving its operands into uniform registers: about
    // 70 cycles each, more than the tensor pipe takes for a 128 x 128 x 16
    // product, measured.)
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_bf16_f32(kPpBM, kPpBN, false, false);  // Q K^T
    constexpr uint32_t idesc_o = idesc_bf16_f32(kPpBM, D, false, true);       // P V, V MN-major
    // Shared-memory descriptors are linear in the address (its low 14 bits
    // hold address / 16, and every operand here lies below 256 KB), so each
    // MMA's descriptor is a base descriptor plus a constant.
    const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + C::kVOff), C::kKVHalf, 1024);
    int kc = 0, vc = 0, units = 0;
    int pl[2] = {0, 0}, ph[2] = {0, 0};  // p_lo, p_hi phases awaited
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, int parity) { return __all_sync(0xffffffffu, pp_wait(bar, parity)); };
    auto commit = [&](uint64_t* bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    // S_t = Q_t K^T, K in stage ks, into columns 128 t
    auto issue_s = [&](int t, int ks) {
      const uint64_t qd = q_desc + (uint64_t)((t * C::kQBytes) >> 4);
      const uint64_t kd = k_desc + (uint64_t)((ks * C::kKVBytes) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma(tmem + (uint32_t)(t * kPpBN), qd + (uint64_t)(((kk >> 2) * C::kQHalf + (kk & 3) * 32) >> 4),
                 kd + (uint64_t)(((kk >> 2) * C::kKVHalf + (kk & 3) * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
      }
      __syncwarp();
    };
    // one half (keys 64 hh ..) of O_t += P_t V, V in stage vs, P_t in columns 128 t + 64 hh .. + 31
    auto issue_pv_half = [&](int t, int vs, int hh, bool acc) {
      const uint64_t vd = v_desc + (uint64_t)((vs * C::kKVBytes) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk)
          tc_mma_tmem_a(tmem + C::kOCol + (uint32_t)(t * 128), tmem + (uint32_t)(t * kPpBN + 64 * hh + (kk - 4 * hh) * 8),
                        vd + (uint64_t)((kk * 16 * 128) >> 4), idesc_o, (acc || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    for (int k = 0; ok; ++k, ++units) {
      int b, seq0, len, qt, g, pr;
      if (!pp_unit<D>(p, smem, k, b, seq0, len, qt, g, pr)) break;
      const int nt = qt + 1;
      if (!(ok = wait_all(&q_full[0], units & 1) && wait_all(&q_full[1], units & 1))) break;
      if (!(ok = wait_all(&k_full[kc % S], (kc / S) & 1))) break;
      tc_fence_after();
      for (int t = 0; t < 2; ++t) {
        issue_s(t, kc % S);
        commit(&s_full[t]);
      }
      commit(&k_empty[kc % S]);
      ++kc;
      if (nt == 1) {
        commit(&q_empty[0]);
        commit(&q_empty[1]);
      }
      for (int j = 0; j < nt && ok; ++j) {
        const bool next = j + 1 < nt;
        if (next && !(ok = wait_all(&k_full[kc % S], (kc / S) & 1))) break;
        const int vs = vc % S;
        if (!(ok = wait_all(&v_full[vs], (vc / S) & 1))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = wait_all(&p_lo[t], pl[t] & 1))) break;
          ++pl[t];
          if (j == 0 && units > 0 && !(ok = wait_all(&o_free[t], (units - 1) & 1))) break;
          tc_fence_after();
          issue_pv_half(t, vs, 0, j > 0);
          if (!(ok = wait_all(&p_hi[t], ph[t] & 1))) break;
          ++ph[t];
          tc_fence_after();
          issue_pv_half(t, vs, 1, true);
          if (j == nt - 1) commit(&o_ready[t]);
          if (next) {  // S_t(j+1), over P_t(j)
            issue_s(t, kc % S);
            commit(&s_full[t]);
            if (j + 1 == nt - 1) commit(&q_empty[t]);
          }
        }
        commit(&v_empty[vs]);
        ++vc;
        if (next) {
          commit(&k_empty[kc % S]);
          ++kc;
        }
      }
    }
    commit(mma_done);  // completes when every MMA issued above has finished
    wait_all(mma_done, 0);
  } else {
    // ----------------------------------------------------- softmax + epilogue
    const int t = warp >> 3, hh = (warp >> 2) & 1, q = warp & 3;
    const int r = q * 32 + lane;  // row within the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t s_addr = lane_base + (uint32_t)(t * kPpBN + 64 * hh);  // this half's 64 score columns
    const uint32_t o_addr = lane_base + (uint32_t)(C::kOCol + t * 128);
    float* xbuf = reinterpret_cast<float*>(smem + C::kXOff) + t * (2 * 2 * kPpBM);
    uint64_t* xbar = &pair[t * 4 + q];  // the partner warps' barrier (a bounded wait, unlike bar.sync)
    int xc = 0;                         // exchanges made (their slot and the barrier phase alternate)
    // this row's value from the partner warp (the other key half); NaN if the partner never came.
    // Every lane of both warps calls it (64 arrivals); it returns with the warp converged, as the
    // warp-collective tcgen05 loads and stores that follow require.
    auto exchange = [&](float v) -> float {
      float* e = xbuf + (xc & 1) * (2 * kPpBM);
      e[hh * kPpBM + r] = v;
      mbar_arrive(xbar);
      const bool came = pp_wait(xbar, xc & 1);
      ++xc;
      const float o = came ? e[(1 - hh) * kPpBM + r] : __int_as_float(0x7fc00000);
      __syncwarp();
      return o;
    };
    const float sl2 = p.scale_log2;
    const bool pos_scale = sl2 > 0.f;
    const float xs = pos_scale ? sl2 : 1.f;  // the scale still to apply to the loaded scores
    int sp = 0, units = 0;
    bool ok = true;
    for (int k = 0; ok; ++k, ++units) {
      int b, seq0, len, qt, g, pr;
      if (!pp_unit<D>(p, smem, k, b, seq0, len, qt, g, pr)) break;
      const int nt = qt + 1;
      const int qpos = qt * kPpBM + r;
      float m_used = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      for (int j = 0; j < nt; ++j, ++sp) {
        // tcgen05.ld/st are warp-collective: every decision that guards them is warp-uniform
        if (!__all_sync(0xffffffffu, pp_wait(&s_full[t], sp & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys 64 hh + 32 c + i of the tile with i <= kmax - 32 c are visible
        const int kmax = min(qpos, len - 1) - j * kPpBN - 64 * hh;
        float x[32];
        auto load_chunk = [&](int c) {
          tmem_ld32(s_addr + 32 * c, x);
          tc_wait_ld();
          const int km = kmax - 32 * c;
          if (!(pos_scale && km >= 31)) {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = i <= km ? (pos_scale ? x[i] : x[i] * sl2) : -INFINITY;
          }
        };
        // the maximum of this half of the row (log2 units, scale applied; -inf if all masked)
        auto half_max = [&]() -> float {
          float m = -INFINITY;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            load_chunk(c);
            float a = fmax3(x[0], x[1], x[2]);
#pragma unroll
            for (int i = 3; i < 31; i += 2) a = fmax3(a, x[i], x[i + 1]);
            m = fmaxf(m, fmaxf(a, x[31]));
          }
          return m * xs;
        };
        uint32_t pk[32];
        auto half_exps = [&]() -> float {
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            load_chunk(c);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float y0, y1, p0, p1;
              fma2(y0, y1, x[2 * i], x[2 * i + 1], xs, -m_used);
              if (kPpPolyEvery > 0 && i % (kPpPolyEvery > 0 ? kPpPolyEvery : 1) == kPpPolyEvery - 1) {  // FMA pipe
                exp2_poly2(y0, y1, p0, p1);
              } else {
                p0 = fast_exp2(y0);
                p1 = fast_exp2(y1);
              }
              if (i & 1)
                add2(s2, s3, p0, p1);
              else
                add2(s0, s1, p0, p1);
              pk[16 * c + i] = pack_bf16x2(p0, p1);
            }
          }
          return (s0 + s1) + (s2 + s3);
        };
        float alpha = 1.f;
        bool rescale = false;
        // a new row maximum m_t: the running maximum moves only when m_t exceeds it by more than 8
        auto take_max = [&](float m_t) {
          if (m_t > m_used + 8.f) {  // first tile: m_used = -inf (its key 0 is visible to every row)
            const float m_new = fmaxf(m_t, m_used);
            alpha = fast_exp2(m_used - m_new);
            rescale = j > 0;
            m_used = m_new;
          }
        };
        if (j == 0) {
          const float mh = half_max();
          take_max(fmaxf(mh, exchange(mh)));
        }
        float sh = half_exps();
        if (j > 0) {
          // every P of the row is at most 2^8 when the sum of each half is;
          // otherwise (or on a NaN) both halves take the row maximum and recompute
          const bool fail = !(sh <= 256.f);
          const float partner_fail = exchange(fail ? 1.f : 0.f);  // every lane exchanges, failing or not
          const bool row_fail = fail || partner_fail != 0.f;
          if (__any_sync(0xffffffffu, row_fail)) {  // the partner warp holds the same rows: it takes this branch too
            const float mh = half_max();
            take_max(fmaxf(mh, exchange(mh)));
            sh = half_exps();
          }
        }
        l = l * alpha + sh;
        // the P V before this tile's S has finished: O_t may be rescaled now
        // (by the first half's warps, before the first half of P V(j) may run)
        if (hh == 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int cb = 0; cb < D; cb += 32) {
            float o[32];
            tmem_ld32(o_addr + cb, o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(o_addr + cb, o);
          }
        }
        tmem_st16_u(s_addr, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tmem_st16_u(s_addr + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(hh == 0 ? &p_lo[t] : &p_hi[t]);
      }
      if (!ok) break;
      // epilogue: O_t / l -> bf16 rows of head g G + 2 pr + t, each half of the warps D / 2 columns
      const float inv_l = 1.f / (l + exchange(l));
      if (!__all_sync(0xffffffffu, pp_wait(&o_ready[t], units & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // this half's D / 2 columns of the row, read from TMEM before O_t is released; the
      // release comes before the global stores (an arrive orders every earlier store of the
      // thread), so the next unit's first P V does not wait for the output rows to drain:
      // 0.4915 -> 0.4874 ms on 4 x 4096 x 32 x 128, same box. (Staging the rows through
      // shared memory so that each store instruction writes whole 128-byte segments, instead
      // of one 16-byte piece of 32 rows, measured 5 % slower.)
      float o[D / 2];
      tmem_ld32(o_addr + hh * (D / 2), *reinterpret_cast<float(*)[32]>(&o[0]));
      if constexpr (D / 2 > 32) tmem_ld32(o_addr + hh * (D / 2) + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(&o_free[t]);
      uint32_t w[D / 4];  // the row's D / 2 outputs, bf16 pairs
#pragma unroll
      for (int i = 0; i < D / 4; ++i) w[i] = pack_bf16x2(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
      const int h = g * p.G + 2 * pr + t;
      // The row's NC chunks of 16 bytes (chunk c: columns 8 c .. 8 c + 7 of this half) are
      // transposed across each group of NC lanes by butterfly shuffles, so that store k of
      // lane j writes chunk j of the group's row k: one store instruction then writes whole
      // rows of this half (32 / NC rows x D bytes) instead of a 16-byte piece of 32 rows.
      constexpr int NC = D / 16;
      const int j = lane & (NC - 1);
#pragma unroll
      for (int m = 1; m < NC; m <<= 1) {
        const bool up = (j & m) != 0;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          if (c & m) continue;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t send = up ? w[4 * c + e] : w[4 * (c | m) + e];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
            if (up)
              w[4 * c + e] = recv;
            else
              w[4 * (c | m) + e] = recv;
          }
        }
      }
      const int gpos = qt * kPpBM + q * 32 + (lane & ~(NC - 1));  // the group's first query row
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        if (gpos + k < len) {
          uint4* drow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                 (((size_t)seq0 + gpos + k) * p.H + h) * D + hh * (D / 2));
          drow[j] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      __syncwarp();  // converged again before the next unit's warp-collective TMEM loads
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPpMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kPpTmemCols);
  }
}

// 2-D bf16 map over the cache viewed as [B * K * S_max, D] rows, box (64
// columns, box_rows rows), 128-byte swizzle (the layout of a loaded tile).
inline bool encode_cache_rows(PfEncodeFn fn, CUtensorMap* map, void* base, uint64_t rows, uint64_t Dd,
                              uint32_t box_rows) {
  cuuint64_t dims[2] = {Dd, rows};
  cuuint64_t strides[1] = {Dd * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Fixed length (cu_seqlens null): q/out [B, S, H, D], k/v [B, S, K, D].
// Varlen: packed q/out [T, H, D], k/v [T, K, D] of B sequences. With caches
// (not null) every key row below min(len, S_max) is written to its slab.
template <int D>
int launch_prefill_pair_d(PfEncodeFn fn, void* out, const void* q, const void* k, const void* v, void* k_cache,
                          void* v_cache, int B, int S, int H, int K, int S_max, float scale, cudaStream_t st, int sms,
                          const int32_t* cu_seqlens = nullptr, int T = 0) {
  using C = PpCfg<D>;
  CUtensorMap tq, tk, tv, tkc128, tvc128, tkc16, tvc16;
  const uint64_t rows = cu_seqlens ? (uint64_t)T : (uint64_t)B * S;
  if (!encode_bsh(fn, &tq, q, rows, H, D, kPpBM) || !encode_bsh(fn, &tk, k, rows, K, D, kPpBN) ||
      !encode_bsh(fn, &tv, v, rows, K, D, kPpBN))
    return GQA_ERR_CUDA;
  if (k_cache) {
    const uint64_t crows = (uint64_t)B * K * S_max;
    if (!encode_cache_rows(fn, &tkc128, k_cache, crows, D, kPpBN) ||
        !encode_cache_rows(fn, &tvc128, v_cache, crows, D, kPpBN) ||
        !encode_cache_rows(fn, &tkc16, k_cache, crows, D, 16) || !encode_cache_rows(fn, &tvc16, v_cache, crows, D, 16))
      return GQA_ERR_CUDA;
  } else {
    tkc128 = tvc128 = tkc16 = tvc16 = tk;  // unused
  }
  static std::atomic<int> configured[64]{};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
  if (dev >= 0 && dev < 64 && configured[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(prefill_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return GQA_ERR_CUDA;
    configured[dev].store(1, std::memory_order_release);
  }
  PairParams p;
  p.out = out;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.S = S;
  p.H = H;
  p.K = K;
  p.G = H / K;
  p.S_max = S_max;
  p.T = T;
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long per_qt = (long long)K * (p.G / 2);
  const long long units = cu_seqlens ? ((long long)T / kPpBM + B) * per_qt
                                     : (long long)B * ((S + kPpBM - 1) / kPpBM) * per_qt;
  const long long grid = std::max<long long>(1, std::min<long long>(units, sms));
  // the unit list holds each CTA's share (at most units / grid + 1 entries) and the entry's fields
  p.ordered = cu_seqlens != nullptr && B <= kPpMaxSeqs && units <= (long long)(kPpListMax - 1) * grid &&
              per_qt < (1ll << 24);
  return launch_kernel(prefill_pair_kernel<D>, (unsigned)grid, kPpThreads, C::kSmemBytes, st, false, tq, tk, tv,
                       tkc128, tvc128, tkc16, tvc16, p);
}

}  // namespace gqa
