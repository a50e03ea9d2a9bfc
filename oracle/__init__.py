"""Float64 CPU oracle for GQA over a KV cache.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers. The CUDA path never imports this package and this package never
imports the CUDA path; the two share no code.

The arithmetic lives in ``gqa_ref.c`` (plain loops in double). This module
only marshals numpy arrays into it, and adds the two pieces that are not
arithmetic: the per-token KV-cache size formula and the KV append (a row
copy).

Page citations (title, section):
  * KV bytes per token S_KV = 2 * L * K * d_k * bytes: "GQA 完全拆解"
    (pinghaoyang.com.cn), sections 解码推理的内存账本 and 主流模型里的 GQA：
    KV 缓存账本 (there the KV-head count is written G); the per-layer element
    count 2 * K * d_k: "分組查詢注意力" (compassingai.com), section 關鍵引數.
  * KV append: "分組查詢注意力", section 技術原理 (each new token writes K and
    V of shape [batch, 1, K, d_k]); "GQA 完全拆解", section 解码推理的内存账本
    (after step t the new K, V row is appended to the cache).
  * 8-bit KV cache: "GQA 完全拆解", section 更进一步的 KV 压缩 (the cache's K and
    V held as INT8 instead of FP16, orthogonal to GQA: GQA reduces the head
    count, quantization the bytes per element) and "LLaMa3与DeepSeek采用的GQA
    技术", deployment advice (an 8-bit KV cache halves its memory again). The
    pages give no scale convention; the reading used here: symmetric int8
    codes in [-127, 127] with one float32 scale per cached row (token and KV
    head), value = code * scale; quantization in float32: scale = amax / 127,
    code = round-half-even(x / scale). Decoding an 8-bit cache is the decode
    of the values it holds.
  * Fused K/V projection: "GQA 完全拆解", section 工程实现：权重布局、repeat 与
    Kernel 融合 (GQA's W_K, W_V are [K, d_k, d_model]; inference engines merge
    them into one W_KV [K, 2 d_k, d_model] so that one GEMM yields K and V).
    The reading: W_KV[g] holds K's d_k rows, then V's; a token's K and V for
    KV head g are W_KV[g] x, written to the cache at the token's key.
  * Varlen prefill: "GQA 完全拆解", section 主流模型里的 GQA：KV 缓存账本
    (continuous batching with the KV cache: requests of different lengths
    batched together); each sequence of a packed batch is prefilled causally
    on its own.
  * Paged KV cache: "分組查詢注意力", section 下游 / 推論引擎與架構 (the
    paged cache manages blocks of the K KV heads, not of the H query heads,
    and each block is broadcast to the group's H/K query heads when it is
    used); "GQA 完全拆解", section 工程实现：权重布局、repeat 与 Kernel 融合 (the
    block layout is organised by KV head) and section 主流模型里的 GQA：KV 缓存账本
    (paging removes allocation fragmentation and is orthogonal to GQA); "GQA"
    (kongchang.com), list of facts (the KV cache is managed in blocks). The
    pages give no block size or table format; the reading used here is a pool
    [num_blocks, K, block_size, d] and a table [B, max_blocks] of physical
    block numbers, logical block i of sequence b holding its keys
    i * block_size .. (i + 1) * block_size - 1. A paged decode is, by that
    definition, the decode of the cache the table gathers.

Parity status: every function is pinned by a CPU test (tests/test_oracle_pins.py,
tests/test_oracle_cache_write_pins.py and the paged, 8-bit, projection and
varlen pin files); nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_ref.c")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")

F32, BF16, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        # -ffp-contract=off: no fused multiply-add, every step rounds as written
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load_library(path: str):
    """Load an oracle build from ``path`` (the tests use this to load mutants)."""
    return _declare(ctypes.CDLL(path))


def _get(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(lib):
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.ref_decode.restype = I
    lib.ref_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, D, I, P, I64, I]
    lib.ref_prefill_causal.restype = I
    lib.ref_prefill_causal.argtypes = [P, P, P, P, I, I, I, I, I, D, I, P, I64, I]
    lib.ref_meanpool.restype = I
    lib.ref_meanpool.argtypes = [P, P, I64, I, I, I64, I]
    lib.ref_decode_int8.restype = I
    lib.ref_decode_int8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, D, I, P, I64, I]
    lib.ref_quantize_int8.restype = None
    lib.ref_quantize_int8.argtypes = [P, P, P, I, I64, I]
    lib.ref_round_bf16.argtypes = [P, P, I64]
    lib.ref_round_f32.argtypes = [P, P, I64]
    return lib


def _threads(nthreads: Optional[int]) -> int:
    if nthreads:
        return int(nthreads)
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"unsupported dtype {a.dtype}: float64, float32 or uint16 (bfloat16 bits)")


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------------------
# sizes

def kv_cache_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_elt: int) -> int:
    """S_KV = 2 * L * K * d_k * bytes (the factor 2: one K row and one V row)."""
    return 2 * layers * kv_heads * head_dim * bytes_per_elt


def kv_cache_elements_per_layer_token(kv_heads: int, head_dim: int) -> int:
    """2 * K * d_k elements per layer and token."""
    return 2 * kv_heads * head_dim


# ---------------------------------------------------------------------------
# arithmetic (float64)

def decode(q, k_cache, v_cache, seqlens, scale: float, sel=None, nthreads=None, lib=None) -> np.ndarray:
    """q [B,H,d], caches [B,K,S_max,d], seqlens [B] -> float64 [B,H,d].

    With ``sel`` (an int array of (b, h) pairs) only those rows are computed and
    the result is [len(sel), d].
    """
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    B, H, d = q.shape
    Bk, K, S_max, dk = k_cache.shape
    assert Bk == B and dk == d and v_cache.shape == k_cache.shape
    dt = _dtype_code(q)
    assert _dtype_code(k_cache) == dt and _dtype_code(v_cache) == dt
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    assert seqlens.shape == (B,)
    if sel is None:
        out = np.empty((B, H, d), dtype=np.float64)
        selp, nsel = None, 0
    else:
        sel = np.ascontiguousarray(sel, dtype=np.int32).reshape(-1, 2)
        out = np.empty((sel.shape[0], d), dtype=np.float64)
        selp, nsel = sel.ctypes.data, sel.shape[0]
    rc = _get(lib).ref_decode(out.ctypes.data, q.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data,
                              seqlens.ctypes.data, B, H, K, S_max, d, float(scale), dt, selp, nsel,
                              _threads(nthreads))
    if rc != 0:
        raise ValueError("oracle: H must be a multiple of K")
    return out


def prefill_causal(q, k, v, scale: float, sel=None, nthreads=None, lib=None) -> np.ndarray:
    """q [B,S,H,d], k/v [B,S,K,d] -> float64 [B,S,H,d]; row i sees keys j <= i.

    With ``sel`` (an int array of (b, i, h) triples) only those rows are
    computed and the result is [len(sel), d].
    """
    q, k, v = _c(q), _c(k), _c(v)
    B, S, H, d = q.shape
    assert k.shape[:2] == (B, S) and k.shape[3] == d and v.shape == k.shape
    K = k.shape[2]
    dt = _dtype_code(q)
    if sel is None:
        out = np.empty((B, S, H, d), dtype=np.float64)
        selp, nsel = None, 0
    else:
        sel = np.ascontiguousarray(sel, dtype=np.int32).reshape(-1, 3)
        out = np.empty((sel.shape[0], d), dtype=np.float64)
        selp, nsel = sel.ctypes.data, sel.shape[0]
    rc = _get(lib).ref_prefill_causal(out.ctypes.data, q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                      B, S, H, K, d, float(scale), dt, selp, nsel, _threads(nthreads))
    if rc != 0:
        raise ValueError("oracle: H must be a multiple of K")
    return out


def meanpool_kv(src, K: int, lib=None) -> np.ndarray:
    """src [outer, H, inner] -> float64 [outer, K, inner], mean over each group's H/K heads."""
    src = _c(src)
    outer, H, inner = src.shape
    out = np.empty((outer, K, inner), dtype=np.float64)
    rc = _get(lib).ref_meanpool(out.ctypes.data, src.ctypes.data, outer, H, K, inner, _dtype_code(src))
    if rc != 0:
        raise ValueError("oracle: H must be a multiple of K")
    return out


def round_to(x: np.ndarray, like_dtype) -> np.ndarray:
    """Round float64 values to float32 or bfloat16 bits (uint16), nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if np.dtype(like_dtype) == np.float32:
        out = np.empty(x.shape, dtype=np.float32)
        _get().ref_round_f32(x.ctypes.data, out.ctypes.data, x.size)
        return out
    if np.dtype(like_dtype) == np.uint16:
        out = np.empty(x.shape, dtype=np.uint16)
        _get().ref_round_bf16(x.ctypes.data, out.ctypes.data, x.size)
        return out
    if np.dtype(like_dtype) == np.float64:
        return x.copy()
    raise TypeError(like_dtype)


def widen(a: np.ndarray) -> np.ndarray:
    """Stored values (float32, float64 or bfloat16 bits) as float64."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ---------------------------------------------------------------------------
# KV append (a row copy)

def kv_append(k_cache, v_cache, k_new, v_new, pos):
    """Return copies of the caches with row pos[b] of every (b, g) set to the new token.

    Positions outside [0, S_max) leave the cache untouched (the CUDA path
    reports them as a device error instead of writing).
    """
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    B, K, S_max, _ = kc.shape
    for b in range(B):
        p = int(pos[b])
        if 0 <= p < S_max:
            kc[b, :, p, :] = k_new[b]
            vc[b, :, p, :] = v_new[b]
    return kc, vc


def prefill_cache_write(k, v, S_max: int, k_cache=None, v_cache=None):
    """k/v [B,S,K,d] -> caches [B,K,S_max,d] with rows 0..S-1 filled (others kept)."""
    B, S, K, d = k.shape
    if k_cache is None:
        k_cache = np.zeros((B, K, S_max, d), dtype=k.dtype)
        v_cache = np.zeros((B, K, S_max, d), dtype=v.dtype)
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    kc[:, :, :S, :] = np.transpose(k, (0, 2, 1, 3))
    vc[:, :, :S, :] = np.transpose(v, (0, 2, 1, 3))
    return kc, vc


# ---------------------------------------------------------------------------
# paged KV cache: a block table over a pool of blocks (index arithmetic only)

def paged_gather(pool, block_table) -> np.ndarray:
    """pool [num_blocks, K, bs, d], block_table [B, max_blocks] -> cache [B, K, max_blocks * bs, d].

    cache[b, g, i * bs + r] = pool[block_table[b, i], g, r]. A table entry
    outside [0, num_blocks) gives NaN rows (no key of a valid length may
    point there).
    """
    pool = _c(pool)
    table = np.ascontiguousarray(block_table, dtype=np.int64)
    nb, K, bs, d = pool.shape
    B, mb = table.shape
    out = np.empty((B, K, mb * bs, d), dtype=pool.dtype)
    nan = np.uint16(0x7FC0) if pool.dtype == np.uint16 else np.nan  # a quiet NaN (bfloat16 bits or float)
    for b in range(B):
        for i in range(mb):
            blk = int(table[b, i])
            if 0 <= blk < nb:
                out[b, :, i * bs:(i + 1) * bs, :] = pool[blk]
            else:
                out[b, :, i * bs:(i + 1) * bs, :] = nan
    return out


def decode_paged(q, k_pool, v_pool, block_table, seqlens, scale: float, sel=None, nthreads=None,
                 lib=None) -> np.ndarray:
    """q [B,H,d], pools [num_blocks,K,bs,d], block_table [B,max_blocks], seqlens [B] -> float64 [B,H,d]
    (or [len(sel), d]): the decode of the cache that the table gathers."""
    return decode(q, paged_gather(k_pool, block_table), paged_gather(v_pool, block_table), seqlens, scale,
                  sel=sel, nthreads=nthreads, lib=lib)


def kv_append_paged(k_pool, v_pool, k_new, v_new, block_table, pos):
    """Return copies of the pools with key pos[b] of every (b, g) set to the new token: block
    block_table[b, pos[b] // bs], row pos[b] % bs. A position outside [0, max_blocks * bs) or a
    table entry outside [0, num_blocks) leaves the pools untouched."""
    kp, vp = np.array(k_pool, copy=True), np.array(v_pool, copy=True)
    nb, K, bs, _ = kp.shape
    B, mb = np.asarray(block_table).shape
    for b in range(B):
        p = int(pos[b])
        if not 0 <= p < mb * bs:
            continue
        blk = int(block_table[b][p // bs])
        if 0 <= blk < nb:
            kp[blk, :, p % bs, :] = k_new[b]
            vp[blk, :, p % bs, :] = v_new[b]
    return kp, vp


# ---------------------------------------------------------------------------
# 8-bit KV cache: codes int8 [..., d], one float32 scale per row

def quantize_int8(x, lib=None):
    """x [..., n] (float64, float32 or bfloat16 bits) -> (codes int8 [..., n], scales float32 [...])."""
    x = _c(x)
    n = x.shape[-1]
    rows = x.size // n if n else 0
    codes = np.empty(x.shape, dtype=np.int8)
    scales = np.empty(x.shape[:-1], dtype=np.float32)
    if rows:
        _get(lib).ref_quantize_int8(codes.ctypes.data, scales.ctypes.data, x.ctypes.data, _dtype_code(x), rows, n)
    return codes, scales


def decode_int8(q, k_codes, k_scales, v_codes, v_scales, seqlens, scale: float, sel=None, nthreads=None,
                lib=None) -> np.ndarray:
    """q [B,H,d]; k/v codes [B,K,S_max,d] int8, scales [B,K,S_max] float32 -> float64 [B,H,d] (or [len(sel), d])."""
    q = _c(q)
    k_codes, v_codes = _c(k_codes).astype(np.int8, copy=False), _c(v_codes).astype(np.int8, copy=False)
    k_scales = np.ascontiguousarray(k_scales, dtype=np.float32)
    v_scales = np.ascontiguousarray(v_scales, dtype=np.float32)
    B, H, d = q.shape
    Bk, K, S_max, dk = k_codes.shape
    assert Bk == B and dk == d and v_codes.shape == k_codes.shape
    assert k_scales.shape == (B, K, S_max) and v_scales.shape == k_scales.shape
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    if sel is None:
        out = np.empty((B, H, d), dtype=np.float64)
        selp, nsel = None, 0
    else:
        sel = np.ascontiguousarray(sel, dtype=np.int32).reshape(-1, 2)
        out = np.empty((sel.shape[0], d), dtype=np.float64)
        selp, nsel = sel.ctypes.data, sel.shape[0]
    rc = _get(lib).ref_decode_int8(out.ctypes.data, q.ctypes.data, k_codes.ctypes.data, k_scales.ctypes.data,
                                   v_codes.ctypes.data, v_scales.ctypes.data, seqlens.ctypes.data, B, H, K, S_max, d,
                                   float(scale), _dtype_code(q), selp, nsel, _threads(nthreads))
    if rc != 0:
        raise ValueError("oracle: H must be a multiple of K")
    return out


def kv_append_int8(k_codes, k_scales, v_codes, v_scales, k_new, v_new, pos, lib=None):
    """Copies of the 8-bit caches with key pos[b] of every (b, g) set to the quantized new token
    (k_new/v_new [B,K,d]); positions outside [0, S_max) leave the caches untouched."""
    kc, ks, vc, vs = (np.array(a, copy=True) for a in (k_codes, k_scales, v_codes, v_scales))
    B, K, S_max, _ = kc.shape
    kq, kqs = quantize_int8(k_new, lib)
    vq, vqs = quantize_int8(v_new, lib)
    for b in range(B):
        p = int(pos[b])
        if 0 <= p < S_max:
            kc[b, :, p], ks[b, :, p] = kq[b], kqs[b]
            vc[b, :, p], vs[b, :, p] = vq[b], vqs[b]
    return kc, ks, vc, vs


# ---------------------------------------------------------------------------
# varlen (packed) causal prefill: the sequences of a continuous batch back to back

def prefill_causal_varlen(q, k, v, cu_seqlens, scale: float, nthreads=None, lib=None) -> np.ndarray:
    """q [T,H,d], k/v [T,K,d] holding B sequences back to back, sequence b being tokens
    cu_seqlens[b] .. cu_seqlens[b+1]-1 -> float64 [T,H,d]: the causal prefill of every sequence on
    its own (a token sees the keys of its own sequence up to itself)."""
    q, k, v = _c(q), _c(k), _c(v)
    T, H, d = q.shape
    out = np.zeros((T, H, d), dtype=np.float64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 > s0:
            out[s0:s1] = prefill_causal(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], scale, nthreads=nthreads,
                                        lib=lib)[0]
    return out


def prefill_cache_write_varlen(k, v, cu_seqlens, S_max: int, k_cache, v_cache):
    """k/v [T,K,d] packed -> copies of the caches [B,K,S_max,d] with rows 0..len_b-1 of sequence b set."""
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n = min(s1 - s0, S_max)
        kc[b, :, :n, :] = np.transpose(k[s0:s0 + n], (1, 0, 2))
        vc[b, :, :n, :] = np.transpose(v[s0:s0 + n], (1, 0, 2))
    return kc, vc


# ---------------------------------------------------------------------------
# fused K/V projection into the cache (a matmul and row placement)

def kv_project(x, w_kv) -> np.ndarray:
    """x [..., d_model], w_kv [K, 2d, d_model] -> float64 [..., K, 2d]: W_KV[g] x for every KV head g
    (the first d of the 2d outputs are K, the rest V)."""
    xf = widen(np.asarray(x))
    wf = widen(np.asarray(w_kv))
    K, two_d, dm = wf.shape
    out = xf.reshape(-1, dm) @ wf.reshape(K * two_d, dm).T  # a library matmul in float64
    return out.reshape(*xf.shape[:-1], K, two_d)


def kv_project_append(k_cache, v_cache, x, w_kv, pos, like_dtype=np.uint16):
    """x [B, T, d_model], w_kv [K, 2d, d_model], pos [B] (or None: 0) -> copies of the caches [B, K, S_max, d]
    with key pos[b] + i of every (b, g) set to the projection of token (b, i), rounded once to the
    cache's type. A sequence whose rows would not fit (pos < 0 or pos + T > S_max) is left untouched."""
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    B, T, _ = np.asarray(x).shape
    K, two_d, _ = np.asarray(w_kv).shape
    d = two_d // 2
    S_max = kc.shape[2]
    kv = round_to(kv_project(x, w_kv), like_dtype)  # [B, T, K, 2d]
    for b in range(B):
        p0 = 0 if pos is None else int(pos[b])
        if p0 < 0 or p0 + T > S_max:
            continue
        kc[b, :, p0:p0 + T, :] = np.transpose(kv[b, :, :, :d], (1, 0, 2))
        vc[b, :, p0:p0 + T, :] = np.transpose(kv[b, :, :, d:], (1, 0, 2))
    return kc, vc
