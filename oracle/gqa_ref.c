/*
 * Float64 CPU oracle for grouped-query attention over a KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. It shares no
 * code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * It is the plain definition written out, deliberately slow: no tiling, no
 * online softmax, no split of the key axis. Inputs are widened exactly to
 * double; every sum runs in double in ascending index order; the softmax is
 * two-pass (max, then exp and sum) with libm exp.
 *
 * Sources (page title, section):
 *  - "分組查詢注意力" (compassingai.com), section 技術原理: query heads are
 *    reshaped [b,s,H,d_k] -> [b,s,K,H/K,d_k]; every group g runs
 *    softmax(Q_group K_g^T / sqrt(d_k)) V_g against its one K/V head.
 *  - "GQA 完全拆解" (pinghaoyang.com.cn), section "GQA：插值在 MHA 与 MQA
 *    之间的分组共享": group g holds the consecutive query heads
 *    (g-1)h/G+1 .. gh/G (1-based, G = number of groups there), so with
 *    0-based indices head h reads KV head h / (H/K).
 *  - same page, section "从'每头一套键值'说起：解码推理的内存账本": at decode
 *    step t the new query Q_t attends to every cached K_1..t, V_1..t, its
 *    own row included.
 *  - "LLaMa3与DeepSeek采用的GQA技术" (CSDN), section 2: scores = q k^T /
 *    sqrt(d_k), softmax, weighted sum of V.
 *  - "分組查詢注意力", section 模型轉換與 Uptraining, and "GQA 完全拆解",
 *    section Uptraining: the K (and V) projection of group g is the
 *    arithmetic mean of the group's H/K source heads.
 *
 * Readings where the pages are silent: a sequence of length 0 gives zeros;
 * the causal mask of prefill lets query row i see keys j <= i (0-based, no
 * offset, no window); the scale is an argument (the pages fix 1/sqrt(d_k)).
 *
 * Parity status: every function here is pinned by tests against closed forms,
 * brute force and independent library routines; see tests/test_oracle_pins.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_F32 0
#define REF_BF16 1
#define REF_F64 2
#define REF_I8 3 /* caches only: int8 codes, one float scale per row of d */

/* exact widening of one stored element to double */
static double widen(const void* base, int dtype, int64_t i) {
  if (dtype == REF_F64) return ((const double*)base)[i];
  if (dtype == REF_F32) return (double)((const float*)base)[i];
  uint32_t u = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ------------------------------------------------------------------------ */
/* rounding of the float64 result to the storage type (round to nearest even) */

/* bfloat16: 8 significant bits, exponent range of float32 (normal min 2^-126,
 * subnormal quantum 2^-133, largest finite 0x7F7F). */
static uint16_t round_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isinf(a)) return sign | 0x7F80;
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);                       /* a = m * 2^e, m in [0.5, 1) */
  int qexp = e - 8;                   /* quantum of an 8-bit significand */
  if (qexp < -133) qexp = -133;       /* subnormal quantum */
  double q = ldexp(1.0, qexp);
  double r = nearbyint(a / q) * q;    /* default rounding mode: nearest-even */
  if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
  float f = (float)r;                 /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

void ref_round_bf16(const double* x, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

void ref_round_f32(const double* x, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = (float)x[i];
}

/* A K or V cache as stored: elements of `dtype`, or int8 codes whose value
 * is code * scales[row] (row = element index / d), exact in double. */
typedef struct {
  const void* base;
  const float* scales;
  int dtype;
  int d;
} kv_src;

static double widen_kv(const kv_src* c, int64_t i) {
  if (c->dtype == REF_I8) return (double)((const int8_t*)c->base)[i] * (double)c->scales[i / c->d];
  return widen(c->base, c->dtype, i);
}

/* ------------------------------------------------------------------------ */
/* attention of one query row against keys 0..n-1 of one KV head            */

/* q: d values at q + q_off; key t: element kv_off + t*kv_stride of k (d values) */
static void attend_row(double* out, const void* q, int64_t q_off, int q_dtype, const kv_src* k, const kv_src* v,
                       int64_t kv_off, int64_t kv_stride, int64_t n, int d, double scale, double* s) {
  if (n <= 0) {
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    return;
  }
  /* scores s_t = scale * sum_i q_i k_{t,i} */
  for (int64_t t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += widen(q, q_dtype, q_off + i) * widen_kv(k, kv_off + t * kv_stride + i);
    s[t] = scale * acc;
  }
  /* two-pass softmax: m = max_t s_t, w_t = exp(s_t - m), Z = sum_t w_t */
  double m = s[0];
  for (int64_t t = 1; t < n; ++t)
    if (s[t] > m) m = s[t];
  double Z = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    s[t] = exp(s[t] - m);
    Z += s[t];
  }
  /* out = sum_t w_t v_t / Z */
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    double w = s[t];
    for (int i = 0; i < d; ++i) out[i] += w * widen_kv(v, kv_off + t * kv_stride + i);
  }
  for (int i = 0; i < d; ++i) out[i] /= Z;
}

/* ------------------------------------------------------------------------ */
/* decode: q [B,H,d], caches [B,K,S_max,d], seqlens [B] -> out [B,H,d]       */

typedef struct {
  double* out;
  const void* q;
  kv_src kc, vc;
  const int32_t* seqlens;
  int B, H, K, S_max, d;
  double scale;
  int dtype; /* of q */
  const int32_t* sel; /* nsel (b, h) pairs, or NULL for every (b, g) unit */
  int64_t nsel;
  int64_t next;       /* work counter, protected by mu */
  pthread_mutex_t mu;
} decode_job;

static int64_t take(pthread_mutex_t* mu, int64_t* next) {
  pthread_mutex_lock(mu);
  int64_t i = (*next)++;
  pthread_mutex_unlock(mu);
  return i;
}

static void decode_head(decode_job* jb, int b, int h, double* dst, double* s) {
  int G = jb->H / jb->K;
  int g = h / G; /* contiguous grouping: head h reads KV head h / (H/K) */
  int64_t n = jb->seqlens[b];
  if (n < 0) n = 0;
  if (n > jb->S_max) n = jb->S_max;
  int64_t q_off = ((int64_t)b * jb->H + h) * jb->d;
  int64_t kv_off = ((int64_t)b * jb->K + g) * jb->S_max * jb->d;
  attend_row(dst, jb->q, q_off, jb->dtype, &jb->kc, &jb->vc, kv_off, jb->d, n, jb->d, jb->scale, s);
}

static void* decode_worker(void* arg) {
  decode_job* jb = (decode_job*)arg;
  double* s = (double*)malloc(sizeof(double) * (size_t)(jb->S_max > 0 ? jb->S_max : 1));
  int G = jb->H / jb->K;
  if (jb->sel) {
    for (;;) {
      int64_t i = take(&jb->mu, &jb->next);
      if (i >= jb->nsel) break;
      decode_head(jb, jb->sel[2 * i], jb->sel[2 * i + 1], jb->out + i * jb->d, s);
    }
  } else {
    /* loop order of the pages: batch, group, head within the group, key */
    for (;;) {
      int64_t u = take(&jb->mu, &jb->next);
      if (u >= (int64_t)jb->B * jb->K) break;
      int b = (int)(u / jb->K), g = (int)(u % jb->K);
      for (int j = 0; j < G; ++j) {
        int h = g * G + j;
        decode_head(jb, b, h, jb->out + ((int64_t)b * jb->H + h) * jb->d, s);
      }
    }
  }
  free(s);
  return NULL;
}

static void run_threads(void* (*fn)(void*), void* arg, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, fn, arg);
  fn(arg);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* Returns 0, or -1 on a shape the method does not define (H % K != 0). With
 * sel == NULL out is [B,H,d]; otherwise out is [nsel, d] for the listed
 * (b, h) pairs. */
int ref_decode(double* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
               int B, int H, int K, int S_max, int d, double scale, int dtype, const int32_t* sel,
               int64_t nsel, int nthreads) {
  if (K <= 0 || H <= 0 || H % K != 0 || d <= 0 || B < 0 || S_max < 0) return -1;
  decode_job jb = {out, q, {k_cache, NULL, dtype, d}, {v_cache, NULL, dtype, d}, seqlens, B, H, K, S_max, d,
                   scale, dtype, sel, nsel, 0};
  pthread_mutex_init(&jb.mu, NULL);
  run_threads(decode_worker, &jb, nthreads);
  pthread_mutex_destroy(&jb.mu);
  return 0;
}

/* The same over an 8-bit cache: k_codes/v_codes [B,K,S_max,d] int8 with one
 * float scale per row (k_scales/v_scales [B,K,S_max]); the cached value is
 * code * scale ("GQA 完全拆解", section 更进一步的 KV 压缩: the cache's K and V
 * held as INT8). q has q_dtype. */
int ref_decode_int8(double* out, const void* q, const int8_t* k_codes, const float* k_scales, const int8_t* v_codes,
                    const float* v_scales, const int32_t* seqlens, int B, int H, int K, int S_max, int d,
                    double scale, int q_dtype, const int32_t* sel, int64_t nsel, int nthreads) {
  if (K <= 0 || H <= 0 || H % K != 0 || d <= 0 || B < 0 || S_max < 0) return -1;
  decode_job jb = {out, q, {k_codes, k_scales, REF_I8, d}, {v_codes, v_scales, REF_I8, d}, seqlens, B, H, K, S_max,
                   d, scale, q_dtype, sel, nsel, 0};
  pthread_mutex_init(&jb.mu, NULL);
  run_threads(decode_worker, &jb, nthreads);
  pthread_mutex_destroy(&jb.mu);
  return 0;
}

/* Symmetric 8-bit quantization of `rows` rows of n elements (x of dtype
 * REF_BF16, REF_F32 or REF_F64 read as float), in float arithmetic as
 * written: amax = max_i |x_i|; scale = amax / 127; code_i = x_i / scale
 * rounded to nearest, ties to even, clamped to [-127, 127]; a row of zeros
 * gets scale 0 and codes 0. The pages name 8-bit KV caches ("GQA 完全拆解",
 * section 更进一步的 KV 压缩; "LLaMa3与DeepSeek采用的GQA技术", deployment
 * advice) without a scale convention; this per-row symmetric one is the
 * reading taken. Float, not double: a code is an integer decided by floating
 * point, and both implementations decide it in the same precision. */
void ref_quantize_int8(int8_t* codes, float* scales, const void* x, int dtype, int64_t rows, int n) {
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
      float a = fabsf((float)widen(x, dtype, r * n + i));
      if (a > amax) amax = a;
    }
    float sc = amax / 127.0f;
    scales[r] = sc;
    for (int i = 0; i < n; ++i) {
      float c = 0.0f;
      if (sc > 0.0f) {
        c = nearbyintf((float)widen(x, dtype, r * n + i) / sc); /* default rounding: nearest, ties to even */
        if (c > 127.0f) c = 127.0f;
        if (c < -127.0f) c = -127.0f;
      }
      codes[r * n + i] = (int8_t)c;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* causal prefill: q [B,S,H,d], k/v [B,S,K,d] -> out [B,S,H,d]; row i sees    */
/* keys j <= i                                                               */

typedef struct {
  double* out;
  const void* q;
  kv_src k, v;
  int B, S, H, K, d;
  double scale;
  int dtype;
  const int32_t* sel; /* nsel (b, i, h) triples, or NULL for all rows */
  int64_t nsel;
  int64_t next;
  pthread_mutex_t mu;
} prefill_job;

static void prefill_row(prefill_job* jb, int b, int i, int h, double* dst, double* s) {
  int G = jb->H / jb->K;
  int g = h / G;
  int64_t q_off = (((int64_t)b * jb->S + i) * jb->H + h) * jb->d;
  int64_t kv_off = ((int64_t)b * jb->S * jb->K + g) * jb->d; /* key j at kv_off + j*K*d */
  attend_row(dst, jb->q, q_off, jb->dtype, &jb->k, &jb->v, kv_off, (int64_t)jb->K * jb->d, (int64_t)i + 1, jb->d,
             jb->scale, s);
}

static void* prefill_worker(void* arg) {
  prefill_job* jb = (prefill_job*)arg;
  double* s = (double*)malloc(sizeof(double) * (size_t)(jb->S > 0 ? jb->S : 1));
  int G = jb->H / jb->K;
  if (jb->sel) {
    for (;;) {
      int64_t r = take(&jb->mu, &jb->next);
      if (r >= jb->nsel) break;
      prefill_row(jb, jb->sel[3 * r], jb->sel[3 * r + 1], jb->sel[3 * r + 2], jb->out + r * jb->d, s);
    }
  } else {
    for (;;) {
      int64_t u = take(&jb->mu, &jb->next);
      if (u >= (int64_t)jb->B * jb->K) break;
      int b = (int)(u / jb->K), g = (int)(u % jb->K);
      for (int j = 0; j < G; ++j) {
        int h = g * G + j;
        for (int i = 0; i < jb->S; ++i)
          prefill_row(jb, b, i, h, jb->out + (((int64_t)b * jb->S + i) * jb->H + h) * jb->d, s);
      }
    }
  }
  free(s);
  return NULL;
}

int ref_prefill_causal(double* out, const void* q, const void* k, const void* v, int B, int S, int H, int K,
                       int d, double scale, int dtype, const int32_t* sel, int64_t nsel, int nthreads) {
  if (K <= 0 || H <= 0 || H % K != 0 || d <= 0 || B < 0 || S < 0) return -1;
  prefill_job jb = {out, q, {k, NULL, dtype, d}, {v, NULL, dtype, d}, B, S, H, K, d, scale, dtype, sel, nsel, 0};
  pthread_mutex_init(&jb.mu, NULL);
  run_threads(prefill_worker, &jb, nthreads);
  pthread_mutex_destroy(&jb.mu);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* MHA -> GQA mean pooling: src [outer, H, inner] -> out [outer, K, inner],  */
/* out[o,g,i] = (sum over the group's H/K heads of src[o, head, i]) / (H/K)  */

int ref_meanpool(double* out, const void* src, int64_t outer, int H, int K, int64_t inner, int dtype) {
  if (K <= 0 || H <= 0 || H % K != 0 || outer < 0 || inner < 0) return -1;
  int G = H / K;
  for (int64_t o = 0; o < outer; ++o)
    for (int g = 0; g < K; ++g)
      for (int64_t i = 0; i < inner; ++i) {
        double acc = 0.0;
        for (int r = 0; r < G; ++r) acc += widen(src, dtype, (o * H + (int64_t)g * G + r) * inner + i);
        out[(o * K + g) * inner + i] = acc / (double)G;
      }
  return 0;
}
