// KV append (one token, and the bulk prompt write used by prefill) and the
// MHA -> GQA mean pooling. All three are pure HBM streams: 16-byte vector
// accesses, grid-stride loops sized to the SM count.
#pragma once

#include "common.cuh"

namespace gqa {

// ---------------------------------------------------------------------------
// gqa_kv_append: k_cache[b, g, pos[b], :] = k_new[b, g, :] (and V).
// One thread per 16-byte chunk of a new row; both caches in one launch.
// With a block table (gqa_kv_append_paged) the caches are pools of
// num_blocks blocks [K, block_size, d], S_max = max_blocks * block_size, and
// key pos[b] of sequence b is row pos[b] % block_size of block
// block_table[b * max_blocks + pos[b] / block_size].
__global__ void kv_append_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                 const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                 const int32_t* __restrict__ pos, int B, int K, int S_max, int chunks_per_row,
                                 const int32_t* __restrict__ block_table, int max_blocks, int block_size,
                                 int num_blocks) {
  const long long per_tensor = (long long)B * K * chunks_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < 2 * per_tensor;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const long long j = is_v ? i - per_tensor : i;
    const int c = (int)(j % chunks_per_row);
    const long long row = j / chunks_per_row;  // b * K + g
    const int b = (int)(row / K), g = (int)(row % K);
    const int p = __ldg(pos + b);
    const bool reporter = c == 0 && !is_v && g == 0;  // one thread per sequence reports
    if (p < 0 || p >= S_max) {
      if (reporter) raise_error(GQA_DEVERR_APPEND_POS);
      continue;
    }
    long long dst_row = row * S_max + p;
    if (block_table != nullptr) {
      const int blk = __ldg(block_table + (size_t)b * max_blocks + p / block_size);
      if ((unsigned)blk >= (unsigned)num_blocks) {
        if (reporter) raise_error(GQA_DEVERR_BLOCK);
        continue;
      }
      dst_row = ((long long)blk * K + g) * block_size + p % block_size;
    }
    const long long dst = dst_row * chunks_per_row + c;
    if (is_v)
      v_cache[dst] = __ldg(v_new + j);
    else
      k_cache[dst] = __ldg(k_new + j);
  }
}

// gqa_kv_append_int8: the new token's K and V rows (bf16, d = 128) quantized
// into the 8-bit cache at key pos[b]: scale = amax / 127, code = x / scale
// rounded to nearest even, clamped to [-127, 127] (a zero row: scale 0,
// codes 0), in float with correctly rounded divisions. One warp per row
// (4 values per lane), K rows then V rows.
__global__ void kv_append_int8_kernel(int8_t* __restrict__ k_codes, float* __restrict__ k_scales,
                                      int8_t* __restrict__ v_codes, float* __restrict__ v_scales,
                                      const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
                                      const int32_t* __restrict__ pos, int B, int K, int S_max) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * K;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < 2 * nrows; r += warps) {
    const bool is_v = r >= nrows;
    const long long row = is_v ? r - nrows : r;  // b * K + g
    const int b = (int)(row / K);
    const int p = __ldg(pos + b);
    if (p < 0 || p >= S_max) {
      if (lane == 0 && !is_v && row % K == 0) raise_error(GQA_DEVERR_APPEND_POS);
      continue;
    }
    const uint2 w = __ldg(reinterpret_cast<const uint2*>((is_v ? v_new : k_new) + row * D) + lane);
    const float x[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y << 16),
                        __uint_as_float(w.y & 0xffff0000u)};
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float sc = __fdiv_rn(amax, 127.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int c = 0;
      if (sc > 0.f) c = min(127, max(-127, __float2int_rn(__fdiv_rn(x[i], sc))));
      packed |= (uint32_t)(uint8_t)(int8_t)c << (8 * i);
    }
    const long long dst = row * S_max + p;
    reinterpret_cast<uint32_t*>((is_v ? v_codes : k_codes) + dst * D)[lane] = packed;
    if (lane == 0) (is_v ? v_scales : k_scales)[dst] = sc;
  }
}

// Prompt write: k [B, S, K, d] -> k_cache [B, K, S_max, d] rows 0..S-1 (and V).
__global__ void kv_write_prompt_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                       const uint4* __restrict__ k, const uint4* __restrict__ v, int B, int S,
                                       int K, int S_max, int chunks_per_row) {
  const long long per_tensor = (long long)B * S * K * chunks_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < 2 * per_tensor;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const long long j = is_v ? i - per_tensor : i;  // index in [B, S, K, chunks]
    const int c = (int)(j % chunks_per_row);
    long long r = j / chunks_per_row;
    const int g = (int)(r % K);
    r /= K;
    const int s = (int)(r % S);
    const int b = (int)(r / S);
    const long long dst = (((long long)b * K + g) * S_max + s) * chunks_per_row + c;
    if (is_v)
      v_cache[dst] = __ldg(v + j);
    else
      k_cache[dst] = __ldg(k + j);
  }
}

// Varlen prompt write: packed k [T, K, d] of B sequences (cu_seqlens) ->
// k_cache [B, K, S_max, d], row t of sequence b at key t (and V). A token's
// sequence is found by binary search in cu_seqlens; rows at or past S_max
// are not written and set GQA_DEVERR_SEQLEN.
__global__ void kv_write_prompt_varlen_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                              const uint4* __restrict__ k, const uint4* __restrict__ v,
                                              const int32_t* __restrict__ cu_seqlens, int B, int T, int K, int S_max,
                                              int chunks_per_row) {
  const long long per_tensor = (long long)T * K * chunks_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < 2 * per_tensor;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const long long j = is_v ? i - per_tensor : i;  // index in [T, K, chunks]
    const int c = (int)(j % chunks_per_row);
    const long long r = j / chunks_per_row;
    const int g = (int)(r % K);
    const int t = (int)(r / K);
    int lo = 0, hi = B;  // the sequence b with cu[b] <= t < cu[b+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(cu_seqlens + mid) <= t) lo = mid;
      else hi = mid;
    }
    const int pos = t - __ldg(cu_seqlens + lo);
    if (pos < 0 || t >= __ldg(cu_seqlens + lo + 1)) continue;  // a token outside every sequence
    if (pos >= S_max) {
      if (c == 0 && g == 0 && !is_v) raise_error(GQA_DEVERR_SEQLEN);
      continue;
    }
    const long long dst = (((long long)lo * K + g) * S_max + pos) * chunks_per_row + c;
    if (is_v)
      v_cache[dst] = __ldg(v + j);
    else
      k_cache[dst] = __ldg(k + j);
  }
}

// ---------------------------------------------------------------------------
// gqa_meanpool_kv: dst[o, g, i] = sum_{r<G} src[o, g*G + r, i] / G.
// The sum runs in double in ascending r and is rounded once to the output
// type, so the result does not depend on the summation schedule.

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
};

__device__ __forceinline__ void widen16(const uint4& v, double (&x)[8], const __nv_bfloat16*) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    x[2 * k] = (double)__uint_as_float(w[k] << 16);
    x[2 * k + 1] = (double)__uint_as_float(w[k] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void widen16(const uint4& v, double (&x)[8], const float*) {
  x[0] = (double)__uint_as_float(v.x);
  x[1] = (double)__uint_as_float(v.y);
  x[2] = (double)__uint_as_float(v.z);
  x[3] = (double)__uint_as_float(v.w);
}

__device__ __forceinline__ uint4 narrow16(const double (&x)[8], const __nv_bfloat16*) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat16 lo = __double2bfloat16(x[2 * k]);
    __nv_bfloat16 hi = __double2bfloat16(x[2 * k + 1]);
    w[k] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 narrow16(const double (&x)[8], const float*) {
  return make_uint4(__float_as_uint(__double2float_rn(x[0])), __float_as_uint(__double2float_rn(x[1])),
                    __float_as_uint(__double2float_rn(x[2])), __float_as_uint(__double2float_rn(x[3])));
}

// Vector path: inner is a multiple of the 16-byte vector width.
template <typename T>
__global__ void meanpool_vec_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src, long long outer, int H,
                                    int K, long long inner_vecs) {
  constexpr int N = Vec<T>::N;
  const int G = H / K;
  const double inv_g = 1.0 / (double)G;
  const bool pow2 = (G & (G - 1)) == 0;
  const long long total = outer * K * inner_vecs;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long iv = i % inner_vecs;
    const long long og = i / inner_vecs;  // o * K + g
    const long long o = og / K;
    const int g = (int)(og % K);
    const uint4* s = src + ((o * H + (long long)g * G) * inner_vecs + iv);
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int r = 0;
    // eight source vectors requested before any is summed (the summation
    // order stays r = 0, 1, ..., G - 1): 0.71 -> 0.76 of the copy bandwidth
    // for 64 -> 8 heads, against four at a time
    for (; r + 8 <= G; r += 8) {
      uint4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __ldg(s + (long long)(r + q) * inner_vecs);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        double x[8];
        widen16(v[q], x, (const T*)nullptr);
#pragma unroll
        for (int k = 0; k < N; ++k) acc[k] += x[k];
      }
    }
    for (; r + 4 <= G; r += 4) {
      uint4 v0 = __ldg(s + (long long)(r + 0) * inner_vecs);
      uint4 v1 = __ldg(s + (long long)(r + 1) * inner_vecs);
      uint4 v2 = __ldg(s + (long long)(r + 2) * inner_vecs);
      uint4 v3 = __ldg(s + (long long)(r + 3) * inner_vecs);
      double x[8];
      widen16(v0, x, (const T*)nullptr);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += x[k];
      widen16(v1, x, (const T*)nullptr);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += x[k];
      widen16(v2, x, (const T*)nullptr);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += x[k];
      widen16(v3, x, (const T*)nullptr);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += x[k];
    }
    for (; r < G; ++r) {
      double x[8];
      widen16(__ldg(s + (long long)r * inner_vecs), x, (const T*)nullptr);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += x[k];
    }
#pragma unroll
    for (int k = 0; k < N; ++k) acc[k] = pow2 ? acc[k] * inv_g : acc[k] / (double)G;
    dst[i] = narrow16(acc, (const T*)nullptr);
  }
}

// Scalar path for inner sizes that are not a multiple of the vector width.
template <typename T>
__global__ void meanpool_scalar_kernel(T* __restrict__ dst, const T* __restrict__ src, long long outer, int H, int K,
                                       long long inner) {
  const int G = H / K;
  const long long total = outer * K * inner;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long ii = i % inner;
    const long long og = i / inner;
    const long long o = og / K;
    const int g = (int)(og % K);
    double acc = 0.0;
    for (int r = 0; r < G; ++r) {
      const T x = src[(o * H + (long long)g * G + r) * inner + ii];
      if constexpr (sizeof(T) == 2)
        acc += (double)__bfloat162float(x);
      else
        acc += (double)x;
    }
    acc = acc / (double)G;
    if constexpr (sizeof(T) == 2)
      dst[i] = __double2bfloat16(acc);
    else
      dst[i] = __double2float_rn(acc);
  }
}

}  // namespace gqa
