/*
 * gqa.h - grouped-query attention (GQA) over a KV cache, for NVIDIA B200
 * (sm_100a). C ABI of libgqa.so.
 *
 * Notation: B batch, H query heads, K KV heads, G = H / K query heads per
 * group, d head dimension, S_max cache capacity in tokens, len_b = seqlens[b].
 * Query head h reads KV head h / G (contiguous grouping): "分組查詢注意力"
 * (compassingai.com), section 技術原理, reshapes Q [b,s,H,d_k] into
 * [b,s,K,H/K,d_k]; "GQA 完全拆解" (pinghaoyang.com.cn), section "GQA：插值在
 * MHA 与 MQA 之间的分组共享", gives group g the consecutive heads
 * (g-1)h/G+1 .. gh/G.
 *
 * Cache layout: [B, K, S_max, d], row-major. Each (b, g) slab is contiguous,
 * rows are d elements ("GQA 完全拆解", section 工程实现, organises the cache
 * as layer x KV head x position; "LLaMa3与DeepSeek采用的GQA技术" (CSDN),
 * section 3, keeps each group's KV contiguous).
 *
 * Conventions shared by every call:
 *  - All pointers are DEVICE pointers unless stated otherwise. The caller
 *    owns every buffer; the library allocates no device memory.
 *  - Every tensor is contiguous and its base address is 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). The return value reports host-side validation and the
 *    kernel launch only. Problems found on the device (an append position
 *    outside the cache, a length outside [0, S_max], a bounded pipeline wait
 *    that expired) never trap: they set bits of a per-device error word that
 *    gqa_get_last_error() reads and clears.
 *  - dtype is the storage type of every floating-point tensor of the call;
 *    outputs use the same type. Arithmetic: float32 accumulation.
 *  - Supported head dimensions: 64 and 128. H must be a multiple of K.
 */
#ifndef GQA_H_
#define GQA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* gqa_stream_t;

typedef enum { GQA_F32 = 0, GQA_BF16 = 1 } gqa_dtype;

typedef enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = -1, /* NULL pointer, negative size, bad dtype, workspace too small */
  GQA_ERR_SHAPE = -2,       /* H % K != 0, d not in {64, 128}, sizes beyond int32 indexing */
  GQA_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
  GQA_ERR_CUDA = -4,        /* a CUDA call or kernel launch failed */
  GQA_ERR_DEVICE = -5,      /* the device error word was set (see GQA_DEVERR_*) */
  GQA_ERR_UNSUPPORTED = -6, /* valid request that this build does not implement (e.g. f32 prefill) */
  GQA_ERR_SCRATCH_LIMIT = -7 /* gqa_decode_noalloc: needs more than GQA_NOALLOC_SCRATCH_BYTES of scratch */
} gqa_status;

/* Bits of the device error word. */
#define GQA_DEVERR_APPEND_POS 0x1u /* gqa_kv_append: pos[b] outside [0, S_max); row not written */
#define GQA_DEVERR_SEQLEN 0x2u     /* gqa_decode: seqlens[b] outside [0, S_max]; out[b] set to zero */
#define GQA_DEVERR_TIMEOUT 0x4u    /* a bounded wait in a pipelined kernel expired; output invalid */
#define GQA_DEVERR_BLOCK 0x8u      /* paged cache: a block-table entry outside [0, num_blocks) was read;
                                      block 0 was used in its place, output invalid */

/*
 * gqa_kv_append - write one new token's K and V rows into the cache.
 *
 * Defined by "分組查詢注意力", section 技術原理 (each new token writes K and V
 * of shape [batch, 1, K, d_k], not [batch, 1, H, d_k]) and "GQA 完全拆解",
 * section 解码推理的内存账本 (after decode step t the new K, V row is appended).
 *
 *   k_cache[b, g, pos[b], :] = k_new[b, g, :]   for every b < B, g < K
 *   v_cache[b, g, pos[b], :] = v_new[b, g, :]
 *
 * k_cache, v_cache : [B, K, S_max, d], written in place (only those rows).
 * k_new, v_new     : [B, K, d].
 * pos              : [B] int32, device. pos[b] is the length of sequence b
 *                    before the append; the decode that follows uses
 *                    seqlens[b] = pos[b] + 1 so the new token sees itself.
 * A position outside [0, S_max) is not written and sets GQA_DEVERR_APPEND_POS.
 */
GQA_API int gqa_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos, int B,
                  int K, int S_max, int d, gqa_dtype dtype, gqa_stream_t stream);

/*
 * gqa_decode_workspace_bytes - device workspace gqa_decode needs for the
 * split-KV partial results of this shape (0 when no split is needed).
 * num_splits as for gqa_decode (0 = automatic). Returns 0 for invalid shapes.
 */
GQA_API size_t gqa_decode_workspace_bytes(int B, int H, int K, int S_max, int d, int num_splits);

/*
 * gqa_decode - one decode step: every query head attends to its group's
 * cached keys and values.
 *
 * Defined by "GQA 完全拆解", section 解码推理的内存账本 (at step t the new Q_t
 * attends to all cached K_1..t, V_1..t) and section "GQA：插值在 MHA 与 MQA
 * 之间的分组共享" (head i of group g uses the group's shared K_g, V_g);
 * "LLaMa3与DeepSeek采用的GQA技术", section 2 (scores = q k^T / sqrt(d_k),
 * softmax, weighted sum of V):
 *
 *   out[b, h, :] = sum_{t < len_b} softmax_t(scale * q[b,h,:] . k[b,g,t,:]) v[b,g,t,:],
 *   g = h / (H / K)
 *
 * out       : [B, H, d], written.
 * q         : [B, H, d].
 * k_cache   : [B, K, S_max, d]; v_cache likewise. Rows t >= len_b are never
 *             read into the result (their contents do not matter).
 * seqlens   : [B] int32, device. len_b == 0 gives out[b] = 0. A value outside
 *             [0, S_max] sets GQA_DEVERR_SEQLEN and gives out[b] = 0.
 * scale     : the score scale, normally 1/sqrt(d).
 * num_splits: how many key-axis partitions per (b, g) (split-KV with a
 *             log-sum-exp combine); 0 picks one from the shape and the GPU.
 * workspace : device scratch of at least gqa_decode_workspace_bytes(...)
 *             bytes for the same shape and num_splits; may be NULL when that
 *             size is 0. Its contents need no initialisation. Two calls that
 *             share a workspace must not overlap on the GPU.
 *
 * The call may be captured into a CUDA graph (stream capture) and replayed:
 * nothing is read back to the host, and the work counter the persistent
 * kernel keeps in the workspace is left reset at the end of every launch.
 * A replay reuses the pointers and sizes of the capture.
 */
GQA_API int gqa_decode(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, int B,
               int H, int K, int S_max, int d, float scale, int num_splits, void* workspace, size_t workspace_bytes,
               gqa_dtype dtype, gqa_stream_t stream);

/*
 * gqa_decode_append - one decode step with the new token's append fused in:
 * the effect of gqa_kv_append(k_cache, v_cache, k_new, v_new, pos, ...)
 * followed by gqa_decode(..., seqlens = pos + 1, ...), in one pass over the
 * cache ("GQA 完全拆解", section 解码推理的内存账本: the new query attends to
 * every cached key including its own, and the new K, V row joins the cache).
 *
 * k_cache, v_cache : [B, K, S_max, d]; row pos[b] of every (b, g) is written.
 * k_new, v_new     : [B, K, d], the new token's K and V.
 * pos              : [B] int32, device: the length of each sequence before
 *                    the append. pos[b] outside [0, S_max) sets
 *                    GQA_DEVERR_APPEND_POS, writes nothing and gives
 *                    out[b] = 0.
 * Everything else as for gqa_decode; the workspace size is
 * gqa_decode_workspace_bytes of the same shape. bf16 runs as one decode
 * kernel (plus the split combine); f32 launches the append first.
 */
GQA_API int gqa_decode_append(void* out, const void* q, void* k_cache, void* v_cache, const void* k_new,
                              const void* v_new, const int32_t* pos, int B, int H, int K, int S_max, int d,
                              float scale, int num_splits, void* workspace, size_t workspace_bytes, gqa_dtype dtype,
                              gqa_stream_t stream);

/*
 * gqa_decode_noalloc - gqa_decode without a caller-supplied workspace.
 *
 * The paper has no counterpart to this call. It is for callers that cannot
 * allocate device memory when they decode, such as a plugin inside a host
 * framework that owns all device memory through its own allocator (a raw
 * cudaMalloc would bypass that allocator's budget), or a latency-critical
 * serving loop that allows no allocation after start-up (cudaMalloc and
 * cudaFree can synchronise the whole device). Such a caller still passes
 * out, q, the caches and seqlens exactly as for gqa_decode.
 *
 * The split-KV partial results go to a scratch array the library holds
 * itself: GQA_NOALLOC_SCRATCH_BYTES of static device memory on every GPU that
 * loads the library, kept until the process exits. The call itself allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *  - A request whose partials need more than GQA_NOALLOC_SCRATCH_BYTES (what
 *    gqa_decode_workspace_bytes reports for the same shape and num_splits)
 *    is rejected with GQA_ERR_SCRATCH_LIMIT before anything is launched; a
 *    smaller num_splits needs less scratch.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current). Under CUDA's lazy
 *    module loading (the default since CUDA 12.2) that lookup may load the
 *    part of the library that holds the array: it reserves the
 *    GQA_NOALLOC_SCRATCH_BYTES and can synchronise the device, as an
 *    allocation would. Make one call per device at start-up, before any
 *    stream capture begins on the device.
 *  - A device reset (cudaDeviceReset) ends the context the address belongs
 *    to. The next call sees that the device's context changed and looks the
 *    address up again (which again loads the module, as above).
 *  - Every call on a device uses the same array, which keeps whatever the
 *    last call left in it. Calls that overlap on the GPU (unordered streams)
 *    race on it and produce wrong results: order them on one stream or with
 *    events. Nothing in it has to start at zero; within one call every
 *    partial is written before it is read.
 *  - Arguments, results and errors are otherwise those of gqa_decode.
 */
#define GQA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
GQA_API int gqa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* seqlens, int B, int H, int K, int S_max, int d, float scale,
                               int num_splits, gqa_dtype dtype, gqa_stream_t stream);

/*
 * Paged KV cache: the paged forms of gqa_kv_append, gqa_decode and
 * gqa_decode_append.
 *
 * "分組查詢注意力", section 下游 / 推論引擎與架構: a paged cache manages blocks
 * of the K KV heads (not of the H query heads), and each block is broadcast
 * to the H/K query heads of its group when it is used; "GQA 完全拆解",
 * section 工程实现：权重布局、repeat 与 Kernel 融合: the block layout is organised
 * by KV head and the kernel broadcasts within the group, and section
 * 主流模型里的 GQA：KV 缓存账本: paging removes allocation fragmentation and is
 * orthogonal to GQA. The pages give no block size or table format; here:
 *
 * k_pool, v_pool : [num_blocks, K, block_size, d]: block n holds block_size
 *                  consecutive keys of one sequence for every KV head.
 * block_table    : [B, max_blocks] int32, device. block_table[b, i] is the
 *                  block holding keys i*block_size .. (i+1)*block_size - 1 of
 *                  sequence b. Entries for keys a call does not touch are
 *                  never read (they may hold anything, e.g. -1). An entry
 *                  that is read and lies outside [0, num_blocks) sets
 *                  GQA_DEVERR_BLOCK: the decode reads block 0 in its place
 *                  (output invalid), the append writes nothing.
 * block_size     : keys per block, a positive multiple of 16.
 * max_blocks     : table row length; the capacity per sequence is
 *                  S_max = max_blocks * block_size, and seqlens / pos are
 *                  checked against it as for the contiguous cache.
 *
 * The results are those of the contiguous calls on the cache the table
 * gathers: cache[b, g, t] = pool[block_table[b, t / block_size], g,
 * t % block_size]. The decode forms are bf16 only (GQA_F32 returns
 * GQA_ERR_UNSUPPORTED); the append takes bf16 or f32. The caller owns the
 * pools, the table and the workspace. Invalid sizes return GQA_ERR_SHAPE.
 */
GQA_API size_t gqa_decode_paged_workspace_bytes(int B, int H, int K, int d, int block_size, int max_blocks,
                                                int num_splits);
GQA_API int gqa_decode_paged(void* out, const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_table, const int32_t* seqlens, int B, int H, int K, int d,
                             int num_blocks, int block_size, int max_blocks, float scale, int num_splits,
                             void* workspace, size_t workspace_bytes, gqa_dtype dtype, gqa_stream_t stream);
GQA_API int gqa_decode_append_paged(void* out, const void* q, void* k_pool, void* v_pool, const void* k_new,
                                    const void* v_new, const int32_t* block_table, const int32_t* pos, int B, int H,
                                    int K, int d, int num_blocks, int block_size, int max_blocks, float scale,
                                    int num_splits, void* workspace, size_t workspace_bytes, gqa_dtype dtype,
                                    gqa_stream_t stream);
GQA_API int gqa_kv_append_paged(void* k_pool, void* v_pool, const void* k_new, const void* v_new,
                                const int32_t* block_table, const int32_t* pos, int B, int K, int d, int num_blocks,
                                int block_size, int max_blocks, gqa_dtype dtype, gqa_stream_t stream);

/*
 * 8-bit KV cache: gqa_kv_append_int8 and gqa_decode_int8.
 *
 * "GQA 完全拆解", section 更进一步的 KV 压缩: the cache's K and V held as INT8
 * instead of FP16, orthogonal to GQA (GQA reduces the head count,
 * quantization the bytes per element); "LLaMa3与DeepSeek采用的GQA技术",
 * deployment advice: an 8-bit KV cache halves its memory again. The pages
 * give no scale convention; here:
 *
 *   value[b, g, t, i] = k_codes[b, g, t, i] * k_scales[b, g, t]   (V likewise)
 *
 * k_codes, v_codes   : [B, K, S_max, d] int8, codes in [-127, 127].
 * k_scales, v_scales : [B, K, S_max] float32, one scale per cached row.
 * d must be 128 and S_max a multiple of 4 (GQA_ERR_UNSUPPORTED /
 * GQA_ERR_SHAPE otherwise).
 *
 * gqa_kv_append_int8 quantizes the new token's rows k_new, v_new ([B, K, d]
 * bfloat16) into key pos[b]: scale = amax / 127 and code = x / scale rounded
 * to nearest (ties to even) and clamped to [-127, 127], in float with
 * correctly rounded divisions (a row of zeros: scale 0, codes 0). pos as for
 * gqa_kv_append (GQA_DEVERR_APPEND_POS outside [0, S_max)).
 *
 * gqa_decode_int8 is gqa_decode over the values the 8-bit cache holds: q and
 * out are [B, H, d] bfloat16, everything else (seqlens, scale, num_splits,
 * the workspace of gqa_decode_int8_workspace_bytes bytes, errors) as for
 * gqa_decode. Rows t >= len_b are never read into the result.
 */
GQA_API size_t gqa_decode_int8_workspace_bytes(int B, int H, int K, int S_max, int d, int num_splits);
GQA_API int gqa_decode_int8(void* out, const void* q, const int8_t* k_codes, const float* k_scales,
                            const int8_t* v_codes, const float* v_scales, const int32_t* seqlens, int B, int H,
                            int K, int S_max, int d, float scale, int num_splits, void* workspace,
                            size_t workspace_bytes, gqa_stream_t stream);
GQA_API int gqa_kv_append_int8(int8_t* k_codes, float* k_scales, int8_t* v_codes, float* v_scales,
                               const void* k_new, const void* v_new, const int32_t* pos, int B, int K, int S_max,
                               int d, gqa_stream_t stream);

/*
 * gqa_prefill_causal - causal self-attention over a whole prompt, and the
 * write of its keys and values into the cache.
 *
 * "GQA 完全拆解", section 解码推理的内存账本 (prefill processes the whole
 * sequence in parallel) and section 质量与速度的实测权衡 (prefill is compute
 * bound and writes the KV once). Causal mask: query row i sees keys j <= i.
 *
 *   out[b, i, h, :] = sum_{j <= i} softmax_j(scale * q[b,i,h,:] . k[b,j,g,:]) v[b,j,g,:]
 *
 * out        : [B, S, H, d], written.
 * q          : [B, S, H, d].
 * k, v       : [B, S, K, d].
 * k_cache,
 * v_cache    : [B, K, S_max, d] or both NULL. When given, rows 0..S-1 of
 *              every (b, g) are set to k[b, :, g, :] / v[b, :, g, :]; other
 *              rows are left as they are. Requires S <= S_max.
 * dtype      : GQA_BF16 only (GQA_F32 returns GQA_ERR_UNSUPPORTED).
 */
GQA_API int gqa_prefill_causal(void* out, const void* q, const void* k, const void* v, void* k_cache, void* v_cache, int B,
                       int S, int H, int K, int S_max, int d, float scale, gqa_dtype dtype, gqa_stream_t stream);

/*
 * gqa_prefill_causal_varlen - gqa_prefill_causal over a packed batch of
 * prompts of different lengths (continuous batching, "GQA 完全拆解", section
 * 主流模型里的 GQA：KV 缓存账本): every sequence is prefilled causally on its own.
 *
 * q, out     : [T, H, d]; k, v : [T, K, d]: the B sequences back to back.
 * cu_seqlens : [B + 1] int32, device: sequence b is rows cu_seqlens[b] ..
 *              cu_seqlens[b+1] - 1 (cu_seqlens[0] = 0, nondecreasing,
 *              cu_seqlens[B] = T). Entries outside [0, T] or decreasing set
 *              GQA_DEVERR_SEQLEN and are clamped into [0, T].
 * k_cache,
 * v_cache    : [B, K, S_max, d] or both NULL. When given, row t of sequence b
 *              is written at key t; rows at or past S_max are not written
 *              and set GQA_DEVERR_SEQLEN.
 * dtype      : GQA_BF16 only (GQA_F32 returns GQA_ERR_UNSUPPORTED).
 */
GQA_API int gqa_prefill_causal_varlen(void* out, const void* q, const void* k, const void* v, void* k_cache,
                                      void* v_cache, const int32_t* cu_seqlens, int B, int T, int H, int K,
                                      int S_max, int d, float scale, gqa_dtype dtype, gqa_stream_t stream);

/*
 * gqa_kv_project_append - the K/V projection of new tokens, written straight
 * into the cache.
 *
 * "GQA 完全拆解", section 工程实现：权重布局、repeat 与 Kernel 融合: GQA's W_K and
 * W_V are [K, d_k, d_model]; inference engines merge them into one
 * W_KV [K, 2 d_k, d_model] so that one GEMM yields K and V. Here:
 *
 *   k_cache[b, g, pos[b] + i, :] = (W_KV[g] x[b, i, :])[0 : d]
 *   v_cache[b, g, pos[b] + i, :] = (W_KV[g] x[b, i, :])[d : 2d]
 *
 * x         : [B, T, d_model] bfloat16: T new tokens per sequence (1 for a
 *             decode step, the prompt for a prefill).
 * w_kv      : [K, 2d, d_model] bfloat16: K's d rows, then V's, per KV head.
 * pos       : [B] int32, device: the key of each sequence's first new token,
 *             or NULL (0 for every sequence). pos[b] < 0 or pos[b] + T >
 *             S_max sets GQA_DEVERR_APPEND_POS and leaves that sequence's
 *             rows unwritten.
 * k_cache,
 * v_cache   : [B, K, S_max, d] bfloat16, written in place (only those rows).
 * workspace : gqa_kv_project_workspace_bytes(...) bytes of device scratch
 *             (0 when the GEMM needs no split of d_model); no initialisation.
 * d is 64 or 128 and d_model a multiple of 64; fp32 accumulation, one
 * rounding to bf16; GQA_BF16 only.
 */
GQA_API size_t gqa_kv_project_workspace_bytes(int B, int T, int K, int d, int d_model);
GQA_API int gqa_kv_project_append(void* k_cache, void* v_cache, const void* x, const void* w_kv, const int32_t* pos,
                                  int B, int T, int K, int S_max, int d, int d_model, void* workspace,
                                  size_t workspace_bytes, gqa_dtype dtype, gqa_stream_t stream);

/*
 * gqa_meanpool_kv - MHA -> GQA conversion by mean pooling of heads.
 *
 * "分組查詢注意力", section 模型轉換與 Uptraining, and "GQA 完全拆解", section
 * Uptraining: the new K (and V) head of group g is the arithmetic mean of the
 * group's H/K original heads; Q is unchanged.
 *
 *   dst[o, g, i] = (1 / G) * sum_{r < G} src[o, g*G + r, i]
 *
 * src : [outer, H, inner]; dst : [outer, K, inner].
 * Projection weights [H, d_k, d_model] use outer = 1, inner = d_k * d_model;
 * per-head tensors [B, H, S, d] use outer = B, inner = S * d.
 * The sum runs in float64 in ascending head order and is rounded once
 * (nearest-even) to dtype, so the result is the correctly rounded mean
 * whenever the float64 sum is exact (always for bf16 inputs within the
 * normal range and G <= 2^16).
 */
GQA_API int gqa_meanpool_kv(void* dst, const void* src, int64_t outer, int H, int K, int64_t inner, gqa_dtype dtype,
                    gqa_stream_t stream);

/*
 * gqa_get_last_error - synchronise `stream`, then read and clear the device
 * error word of the current device. Returns GQA_OK when it was clear,
 * GQA_ERR_DEVICE when any bit was set (bits stored to *bits if bits != NULL;
 * bits is a HOST pointer), GQA_ERR_CUDA if the synchronisation failed.
 */
GQA_API int gqa_get_last_error(gqa_stream_t stream, uint32_t* bits);

/* Human-readable name of a gqa_status value (static storage). */
GQA_API const char* gqa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H_ */
