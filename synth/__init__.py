"""Seeded synthetic inputs (numbers only; none of the attention arithmetic).

Both the CUDA path and the float64 oracle are fed from here, so that they see
identical input bytes while sharing no code. The generator is defined in
``gen.c`` (splitmix64 counter stream, Box-Muller normals). bfloat16 data is
held on the host as ``numpy.uint16`` bit patterns.

The workloads are the Llama-shaped decode and prefill problems of the GQA
pages: Llama-3-8B (32 query heads, 8 KV heads, head dim 128, "GQA 完全拆解",
KV-cache ledger section), the 70B shape with 64 query heads over 8 KV heads
("分組查詢注意力", key-parameters section), and 128K-token contexts (same
ledger section). Every value is N(0, 1).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")

F32, BF16, F64 = 0, 1, 2
SEED_BASE = 0x6A510000
STREAM_Q, STREAM_K, STREAM_V, STREAM_LENS, STREAM_KNEW, STREAM_VNEW, STREAM_BLOCKS = 1, 2, 3, 4, 5, 6, 7
STREAM_K8, STREAM_V8, STREAM_KSCALE, STREAM_VSCALE = 10, 11, 12, 13


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_stream_key.restype = ctypes.c_uint64
        lib.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_draw.restype = ctypes.c_uint64
        lib.synth_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_int]
        lib.synth_cache.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_int64,
                                    ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                    ctypes.c_int]
        lib.synth_uniform_int.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64,
                                          ctypes.c_int32, ctypes.c_int32]
        lib.synth_int8_cache.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                         ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_int64, ctypes.c_float, ctypes.c_float]
        _lib = lib
    return _lib


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _np_dtype(dtype: int):
    return {F32: np.float32, BF16: np.uint16, F64: np.float64}[dtype]


def stream_key(seed: int, stream: int) -> int:
    return int(_get().synth_stream_key(seed, stream))


def draw(key: int, i: int) -> int:
    return int(_get().synth_draw(key, i))


def normal(shape, dtype: int, seed: int, stream: int, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=_np_dtype(dtype))
    if out.size:
        _get().synth_normal(out.ctypes.data, dtype, stream_key(seed, stream), start, out.size, host_threads())
    return out


def cache(units: int, S_max: int, d: int, dtype: int, seed: int, stream: int,
          lens: Optional[np.ndarray] = None, units_per_len: int = 1) -> np.ndarray:
    """[units, S_max, d] cache; rows at or past lens[u // units_per_len] are quiet NaN."""
    out = np.empty((units, S_max, d), dtype=_np_dtype(dtype))
    lp = None
    if lens is not None:
        lens = np.ascontiguousarray(lens, dtype=np.int32)
        lp = lens.ctypes.data
    if out.size:
        _get().synth_cache(out.ctypes.data, dtype, stream_key(seed, stream), units, S_max, d, lp,
                           units_per_len, host_threads())
    return out


def uniform_int(n: int, lo: int, hi: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    if n:
        _get().synth_uniform_int(out.ctypes.data, stream_key(seed, stream), n, lo, hi)
    return out


# --------------------------------------------------------------------------
# workloads


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    H: int
    K: int
    d: int
    S_max: int
    dtype: int
    seed: int
    lens: tuple = ()          # () -> every sequence has length S_max
    len_range: tuple = ()     # (lo, hi) -> uniform integers drawn from the seed
    append: bool = False      # one kv_append of the last token per step

    @property
    def G(self) -> int:
        return self.H // self.K

    @property
    def elt(self) -> int:
        return 4 if self.dtype == F32 else 2


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    S: int
    H: int
    K: int
    d: int
    dtype: int
    seed: int


DECODE_WORKLOADS = {
    "tiny_decode_b1_h8_k2_d64_s128_f32": DecodeShape(
        "tiny_decode_b1_h8_k2_d64_s128_f32", 1, 8, 2, 64, 128, F32, SEED_BASE + 0),
    "llama3_8b_decode_b8_h32_k8_d128_s8192": DecodeShape(
        "llama3_8b_decode_b8_h32_k8_d128_s8192", 8, 32, 8, 128, 8192, BF16, SEED_BASE + 1, append=True),
    "ragged_70b_decode_b32_h64_k8_d128_s1k_16k": DecodeShape(
        "ragged_70b_decode_b32_h64_k8_d128_s1k_16k", 32, 64, 8, 128, 16384, BF16, SEED_BASE + 2,
        len_range=(1024, 16384)),
    "long_ctx_gqa_b1_h64_k8_d128_s131072": DecodeShape(
        "long_ctx_gqa_b1_h64_k8_d128_s131072", 1, 64, 8, 128, 131072, BF16, SEED_BASE + 3),
    "long_ctx_mqa_b1_h64_k1_d128_s131072": DecodeShape(
        "long_ctx_mqa_b1_h64_k1_d128_s131072", 1, 64, 1, 128, 131072, BF16, SEED_BASE + 3),
}

PREFILL_WORKLOADS = {
    "causal_prefill_b4_s4096_h32_k8_d128": PrefillShape(
        "causal_prefill_b4_s4096_h32_k8_d128", 4, 4096, 32, 8, 128, BF16, SEED_BASE + 4),
}


def seqlens_for(w: DecodeShape) -> np.ndarray:
    if w.lens:
        return np.asarray(w.lens, dtype=np.int32)
    if w.len_range:
        return uniform_int(w.B, w.len_range[0], w.len_range[1], w.seed, STREAM_LENS)
    return np.full(w.B, w.S_max, dtype=np.int32)


def decode_inputs(w: DecodeShape) -> dict:
    """q [B,H,d], k/v cache [B,K,S_max,d] (NaN past each length), seqlens [B];
    with ``append``: k_new/v_new [B,K,d] and pos [B] = seqlens - 1."""
    lens = seqlens_for(w)
    out = {
        "q": normal((w.B, w.H, w.d), w.dtype, w.seed, STREAM_Q),
        "k_cache": cache(w.B * w.K, w.S_max, w.d, w.dtype, w.seed, STREAM_K, lens, w.K).reshape(
            w.B, w.K, w.S_max, w.d),
        "v_cache": cache(w.B * w.K, w.S_max, w.d, w.dtype, w.seed, STREAM_V, lens, w.K).reshape(
            w.B, w.K, w.S_max, w.d),
        "seqlens": lens,
    }
    if w.append:
        out["k_new"] = normal((w.B, w.K, w.d), w.dtype, w.seed, STREAM_KNEW)
        out["v_new"] = normal((w.B, w.K, w.d), w.dtype, w.seed, STREAM_VNEW)
        out["pos"] = (lens - 1).astype(np.int32)
    return out


def prefill_inputs(w: PrefillShape) -> dict:
    """q [B,S,H,d], k/v [B,S,K,d]."""
    return {
        "q": normal((w.B, w.S, w.H, w.d), w.dtype, w.seed, STREAM_Q),
        "k": normal((w.B, w.S, w.K, w.d), w.dtype, w.seed, STREAM_K),
        "v": normal((w.B, w.S, w.K, w.d), w.dtype, w.seed, STREAM_V),
    }


# --------------------------------------------------------------------------
# paged caches: the same seeded cache values, scattered over a pool of blocks


@dataclasses.dataclass(frozen=True)
class PagedShape:
    name: str
    base: str          # the DecodeShape whose values are paged
    block_size: int    # keys per block
    spare_blocks: int  # pool blocks no sequence points to (NaN)


PAGED_WORKLOADS = {
    "paged_llama3_8b_decode_b8_h32_k8_d128_s8192_bs16": PagedShape(
        "paged_llama3_8b_decode_b8_h32_k8_d128_s8192_bs16", "llama3_8b_decode_b8_h32_k8_d128_s8192", 16, 64),
    "paged_ragged_70b_decode_b32_h64_k8_d128_s1k_16k_bs64": PagedShape(
        "paged_ragged_70b_decode_b32_h64_k8_d128_s1k_16k_bs64", "ragged_70b_decode_b32_h64_k8_d128_s1k_16k", 64, 64),
    # multi-query attention (G = 64, the tensor-core wide path) over a paged 128K-token context
    "paged_long_ctx_mqa_b1_h64_k1_d128_s131072_bs16": PagedShape(
        "paged_long_ctx_mqa_b1_h64_k1_d128_s131072_bs16", "long_ctx_mqa_b1_h64_k1_d128_s131072", 16, 64),
}


def permutation(n: int, seed: int, stream: int) -> np.ndarray:
    """A uniformly random permutation of 0..n-1 (Fisher-Yates over the counter stream)."""
    key = stream_key(seed, stream)
    perm = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = draw(key, i) % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def page(k_cache: np.ndarray, v_cache: np.ndarray, lens: np.ndarray, block_size: int, spare_blocks: int,
         seed: int, append_row: bool = False) -> dict:
    """Scatter caches [B,K,S_max,d] into pools [num_blocks,K,block_size,d] at random physical blocks.

    Sequence b gets ceil(n_b / block_size) blocks, n_b = lens[b] (+1 with ``append_row``: the block of
    row lens[b] is mapped as well); its other table entries are -1. Pool blocks that no entry points to
    hold NaN. Returns k_pool, v_pool, block_table [B, max_blocks] int32.
    """
    B, K, S_max, d = k_cache.shape
    assert S_max % block_size == 0
    mb = S_max // block_size
    n = np.minimum(np.asarray(lens, dtype=np.int64) + (1 if append_row else 0), S_max)
    need = (n + block_size - 1) // block_size
    nb = int(need.sum()) + spare_blocks
    perm = permutation(nb, seed, STREAM_BLOCKS)
    table = np.full((B, mb), -1, dtype=np.int32)
    nan = np.uint16(0x7FC0) if k_cache.dtype == np.uint16 else np.nan
    k_pool = np.full((nb, K, block_size, d), nan, dtype=k_cache.dtype)
    v_pool = np.full((nb, K, block_size, d), nan, dtype=v_cache.dtype)
    nxt = 0
    for b in range(B):
        for i in range(int(need[b])):
            blk = int(perm[nxt])
            nxt += 1
            table[b, i] = blk
            k_pool[blk] = k_cache[b, :, i * block_size:(i + 1) * block_size, :]
            v_pool[blk] = v_cache[b, :, i * block_size:(i + 1) * block_size, :]
    return {"k_pool": k_pool, "v_pool": v_pool, "block_table": table}


def paged_inputs(pw: PagedShape) -> dict:
    """decode_inputs of the base workload, plus its caches paged (k_pool, v_pool, block_table)."""
    w = DECODE_WORKLOADS[pw.base]
    inp = decode_inputs(w)
    lens = inp["pos"] if w.append else inp["seqlens"]
    inp.update(page(inp["k_cache"], inp["v_cache"], lens, pw.block_size, pw.spare_blocks, w.seed,
                    append_row=w.append))
    return inp


# --------------------------------------------------------------------------
# 8-bit caches: random codes and per-row scales (no quantizer here: the codes
# are data, the scales are in the range a row of N(0, 1) values would get)


def int8_cache(units: int, S_max: int, d: int, seed: int, stream_codes: int, stream_scales: int,
               lens: Optional[np.ndarray] = None, units_per_len: int = 1, lo: float = 0.015, hi: float = 0.035):
    """(codes int8 [units, S_max, d] uniform over [-127, 127], scales float32 [units, S_max] uniform
    over [lo, hi)); rows at or past lens[u // units_per_len] hold code -128 and a NaN scale."""
    codes = np.empty((units, S_max, d), dtype=np.int8)
    scales = np.empty((units, S_max), dtype=np.float32)
    lp = None
    if lens is not None:
        lens = np.ascontiguousarray(lens, dtype=np.int32)
        lp = lens.ctypes.data
    if codes.size:
        _get().synth_int8_cache(codes.ctypes.data, scales.ctypes.data, stream_key(seed, stream_codes),
                                stream_key(seed, stream_scales), units, S_max, d, lp, units_per_len, lo, hi)
    return codes, scales


INT8_WORKLOADS = {
    "int8_llama3_8b_decode_b8_h32_k8_d128_s8192": "llama3_8b_decode_b8_h32_k8_d128_s8192",
    "int8_ragged_70b_decode_b32_h64_k8_d128_s1k_16k": "ragged_70b_decode_b32_h64_k8_d128_s1k_16k",
}


def int8_inputs(name: str) -> dict:
    """q [B,H,d] (the base workload's), 8-bit caches of the base workload's shape and lengths:
    k_codes/v_codes [B,K,S_max,d] int8, k_scale/v_scale [B,K,S_max] float32, seqlens [B]."""
    w = DECODE_WORKLOADS[INT8_WORKLOADS[name]]
    lens = seqlens_for(w)
    kc, ks = int8_cache(w.B * w.K, w.S_max, w.d, w.seed, STREAM_K8, STREAM_KSCALE, lens, w.K)
    vc, vs = int8_cache(w.B * w.K, w.S_max, w.d, w.seed, STREAM_V8, STREAM_VSCALE, lens, w.K)
    shp = (w.B, w.K, w.S_max)
    return {"q": normal((w.B, w.H, w.d), BF16, w.seed, STREAM_Q), "k_codes": kc.reshape(*shp, w.d),
            "k_scale": ks.reshape(shp), "v_codes": vc.reshape(*shp, w.d), "v_scale": vs.reshape(shp),
            "seqlens": lens}


# --------------------------------------------------------------------------
# varlen prefill: a continuous batch of prompts of different lengths, packed


@dataclasses.dataclass(frozen=True)
class VarlenShape:
    name: str
    B: int
    H: int
    K: int
    d: int
    len_range: tuple  # prompt lengths uniform in [lo, hi]
    S_max: int        # cache capacity per sequence
    seed: int


VARLEN_WORKLOADS = {
    "varlen_prefill_b8_h32_k8_d128_s256_4k": VarlenShape(
        "varlen_prefill_b8_h32_k8_d128_s256_4k", 8, 32, 8, 128, (256, 4096), 4096, SEED_BASE + 5),
}


def varlen_inputs(w: VarlenShape) -> dict:
    """lens [B], cu_seqlens [B+1], q [T,H,d], k/v [T,K,d] (bf16, T = sum of lens)."""
    lens = uniform_int(w.B, w.len_range[0], w.len_range[1], w.seed, STREAM_LENS)
    cu = np.zeros(w.B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    T = int(cu[-1])
    return {"lens": lens, "cu_seqlens": cu, "q": normal((T, w.H, w.d), BF16, w.seed, STREAM_Q),
            "k": normal((T, w.K, w.d), BF16, w.seed, STREAM_K), "v": normal((T, w.K, w.d), BF16, w.seed, STREAM_V)}


# --------------------------------------------------------------------------
# fused K/V projection: hidden states and a merged W_KV of the Llama-3-8B shape


@dataclasses.dataclass(frozen=True)
class ProjShape:
    name: str
    B: int
    T: int        # new tokens per sequence (1: a decode step; the prompt length: a prefill)
    K: int
    d: int
    d_model: int
    S_max: int
    seed: int


PROJ_WORKLOADS = {
    "kv_proj_decode_b8_t1_k8_d128_dm4096": ProjShape("kv_proj_decode_b8_t1_k8_d128_dm4096", 8, 1, 8, 128, 4096,
                                                     8192, SEED_BASE + 6),
    "kv_proj_prefill_b4_t4096_k8_d128_dm4096": ProjShape("kv_proj_prefill_b4_t4096_k8_d128_dm4096", 4, 4096, 8,
                                                         128, 4096, 4096, SEED_BASE + 7),
}


def proj_inputs(w: ProjShape) -> dict:
    """x [B, T, d_model] ~ N(0, 1), w_kv [K, 2d, d_model] ~ N(0, 1/d_model) (bf16), pos [B]: the key of each
    sequence's first new token (decode: len - 1 of a full cache; prefill: 0)."""
    x = normal((w.B, w.T, w.d_model), BF16, w.seed, STREAM_Q)
    wf = normal((w.K, 2 * w.d, w.d_model), F32, w.seed, STREAM_K) / np.float32(np.sqrt(w.d_model))
    wb = (wf.view(np.uint32) + 0x7FFF + ((wf.view(np.uint32) >> 16) & 1)) >> 16  # float32 -> bf16 bits, nearest even
    pos = np.full(w.B, w.S_max - w.T, dtype=np.int32)
    return {"x": x, "w_kv": wb.astype(np.uint16), "pos": pos}
