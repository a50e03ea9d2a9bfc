/*
 * Seeded synthetic inputs for the GQA kernels and for the float64 oracle.
 *
 * This module only draws numbers. It holds none of the attention arithmetic,
 * so the CUDA path and the oracle can both be fed from it without sharing any
 * of the method.
 *
 * Generator (counter based, so any slice can be drawn on any thread):
 *   key(seed, stream) = splitmix64 output number `stream` of the sequence
 *                       whose state starts at `seed`
 *   x(key, i)         = splitmix64 output number i of the sequence whose
 *                       state starts at `key` (i = 0, 1, ...)
 *   normal(key, 2j), normal(key, 2j+1) = Box-Muller pair from
 *       u1 = ((x(key,2j)   >> 11) + 1) * 2^-53   in (0, 1]
 *       u2 =  (x(key,2j+1) >> 11)      * 2^-53   in [0, 1)
 *       r  = sqrt(-2 ln u1), theta = 2 pi u2
 *       even index -> r cos(theta), odd index -> r sin(theta)
 *   float32 value = the double rounded to nearest (C cast)
 *   bfloat16 value = that float32 rounded to nearest-even on its top 16 bits
 *   uniform integer in [lo, hi] = lo + x(key, i) mod (hi - lo + 1)
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_F32 0
#define SYNTH_BF16 1
#define SYNTH_F64 2

static const uint64_t GOLDEN_GAMMA = 0x9E3779B97F4A7C15ULL;

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t stream) { return draw(seed, stream); }

uint64_t synth_draw(uint64_t key, uint64_t i) { return draw(key, i); }

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline void store(void* out, int dtype, uint64_t k, double z) {
  if (dtype == SYNTH_F64) {
    ((double*)out)[k] = z;
  } else if (dtype == SYNTH_F32) {
    ((float*)out)[k] = (float)z;
  } else {
    ((uint16_t*)out)[k] = f32_to_bf16_rne((float)z);
  }
}

/* normals for indices [start, start + count) written to out[0 .. count) */
static void normal_range(void* out, int dtype, uint64_t key, uint64_t start, uint64_t count,
                         uint64_t out_off) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t i = start;
  uint64_t end = start + count;
  while (i < end) {
    uint64_t j = i >> 1;
    double u1 = (double)((draw(key, 2 * j) >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(draw(key, 2 * j + 1) >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double th = two_pi * u2;
    if ((i & 1) == 0) {
      store(out, dtype, out_off + (i - start), r * cos(th));
      if (i + 1 < end) store(out, dtype, out_off + (i + 1 - start), r * sin(th));
      i += 2;
    } else {
      store(out, dtype, out_off + (i - start), r * sin(th));
      i += 1;
    }
  }
}

typedef struct {
  void* out;
  int dtype;
  uint64_t key;
  uint64_t start;
  uint64_t lo, hi; /* slice of [0, count) owned by this thread */
} normal_job;

static void* normal_worker(void* arg) {
  normal_job* jb = (normal_job*)arg;
  if (jb->hi > jb->lo) normal_range(jb->out, jb->dtype, jb->key, jb->start + jb->lo, jb->hi - jb->lo, jb->lo);
  return NULL;
}

/* out[k] = normal(key, start + k) for k < count, using up to nthreads threads */
void synth_normal(void* out, int dtype, uint64_t key, uint64_t start, uint64_t count, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (count < (1u << 16)) nthreads = 1;
  pthread_t th[256];
  normal_job jobs[256];
  uint64_t per = (count + nthreads - 1) / nthreads;
  per += per & 1; /* keep Box-Muller pairs on one thread */
  for (int t = 0; t < nthreads; ++t) {
    uint64_t lo = (uint64_t)t * per;
    uint64_t hi = lo + per;
    if (lo > count) lo = count;
    if (hi > count) hi = count;
    jobs[t] = (normal_job){out, dtype, key, start, lo, hi};
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, normal_worker, &jobs[t]);
  normal_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

typedef struct {
  void* out;
  int dtype;
  uint64_t key;
  int64_t S_max, d;
  const int32_t* lens;
  int64_t units_per_len;
  int64_t u_lo, u_hi;
} cache_job;

static void* cache_worker(void* arg) {
  cache_job* jb = (cache_job*)arg;
  size_t esz = jb->dtype == SYNTH_F64 ? 8 : (jb->dtype == SYNTH_F32 ? 4 : 2);
  for (int64_t u = jb->u_lo; u < jb->u_hi; ++u) {
    int64_t len = jb->S_max;
    if (jb->lens) {
      len = jb->lens[u / jb->units_per_len];
      if (len < 0) len = 0;
      if (len > jb->S_max) len = jb->S_max;
    }
    uint64_t base = (uint64_t)u * jb->S_max * jb->d;
    if (len > 0) normal_range(jb->out, jb->dtype, jb->key, base, (uint64_t)len * jb->d, base);
    /* rows at or past the sequence length hold a quiet-NaN sentinel */
    uint64_t pad = (uint64_t)(jb->S_max - len) * jb->d;
    char* p = (char*)jb->out + (base + (uint64_t)len * jb->d) * esz;
    for (uint64_t k = 0; k < pad; ++k) {
      if (jb->dtype == SYNTH_F64) {
        uint64_t b = 0x7FF8000000000000ULL;
        memcpy(p + k * 8, &b, 8);
      } else if (jb->dtype == SYNTH_F32) {
        uint32_t b = 0x7FC00000u;
        memcpy(p + k * 4, &b, 4);
      } else {
        uint16_t b = 0x7FC0;
        memcpy(p + k * 2, &b, 2);
      }
    }
  }
  return NULL;
}

/*
 * A cache tensor [units, S_max, d]: element (u, t, c) takes normal index
 * (u * S_max + t) * d + c, so its value does not depend on the lengths.
 * Rows t >= lens[u / units_per_len] are filled with a quiet NaN. lens may be
 * NULL (every row drawn).
 */
void synth_cache(void* out, int dtype, uint64_t key, int64_t units, int64_t S_max, int64_t d,
                 const int32_t* lens, int64_t units_per_len, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads > units) nthreads = (int)units;
  if (units_per_len < 1) units_per_len = 1;
  pthread_t th[256];
  cache_job jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = (cache_job){out, dtype, key, S_max, d, lens, units_per_len,
                          units * t / nthreads, units * (t + 1) / nthreads};
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, cache_worker, &jobs[t]);
  if (nthreads > 0) cache_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* out[i] = lo + draw(key, i) mod (hi - lo + 1) */
void synth_uniform_int(int32_t* out, uint64_t key, int64_t n, int32_t lo, int32_t hi) {
  uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)((int64_t)lo + (int64_t)(draw(key, (uint64_t)i) % span));
}

/* 8-bit cache rows: codes uniform over [-127, 127] (one draw each, element
 * (u, t, c) at index (u * S_max + t) * d + c), one scale per row uniform
 * over [lo, hi) (row index u * S_max + t of a second stream); rows at or past
 * lens[u / units_per_len] get code -128 and a quiet-NaN scale. */
void synth_int8_cache(int8_t* codes, float* scales, uint64_t key_codes, uint64_t key_scales, int64_t units,
                      int64_t S_max, int64_t d, const int32_t* lens, int64_t units_per_len, float lo, float hi) {
  const float qnan = __builtin_nanf("");
  for (int64_t u = 0; u < units; ++u) {
    const int64_t n = lens ? (int64_t)lens[u / units_per_len] : S_max;
    for (int64_t t = 0; t < S_max; ++t) {
      const uint64_t row = (uint64_t)(u * S_max + t);
      int8_t* dst = codes + row * (uint64_t)d;
      if (t >= n) {
        for (int64_t c = 0; c < d; ++c) dst[c] = (int8_t)-128;
        scales[row] = qnan;
        continue;
      }
      for (int64_t c = 0; c < d; ++c) dst[c] = (int8_t)((int)(draw(key_codes, row * (uint64_t)d + c) % 255u) - 127);
      scales[row] = lo + (hi - lo) * (float)((double)(draw(key_scales, row) >> 11) * 0x1.0p-53);
    }
  }
}
