"""ctypes binding of libgqa.so (include/gqa.h), same names as the C ABI.

Argument marshalling only: each function takes torch tensors that already
live on the GPU, checks their shapes against one another, and passes raw
pointers, sizes and the current CUDA stream to the library. Every step of the
computation runs in the library's CUDA kernels; there is no other code path.
If the library is missing the import fails with an error naming the build
command.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgqa.so")

GQA_F32, GQA_BF16 = 0, 1
GQA_OK = 0
GQA_ERR_DEVICE = -5
GQA_ERR_UNSUPPORTED = -6
GQA_DEVERR_APPEND_POS, GQA_DEVERR_SEQLEN, GQA_DEVERR_TIMEOUT, GQA_DEVERR_BLOCK = 0x1, 0x2, 0x4, 0x8

GQA_ERR_SCRATCH_LIMIT = -7
GQA_NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024

EXPORTED = ("gqa_kv_append", "gqa_decode_workspace_bytes", "gqa_decode", "gqa_decode_append", "gqa_decode_noalloc",
            "gqa_decode_paged_workspace_bytes", "gqa_decode_paged", "gqa_decode_append_paged", "gqa_kv_append_paged",
            "gqa_decode_int8_workspace_bytes", "gqa_decode_int8", "gqa_kv_append_int8", "gqa_prefill_causal_varlen",
            "gqa_kv_project_workspace_bytes", "gqa_kv_project_append",
            "gqa_prefill_causal", "gqa_meanpool_kv", "gqa_get_last_error", "gqa_status_string")


class GqaError(RuntimeError):
    def __init__(self, fn: str, status: int, bits: int = 0):
        self.status, self.bits = status, bits
        name = _lib.gqa_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn}: {name} ({status})" + (f", device error bits 0x{bits:x}" if bits else ""))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.gqa_kv_append.restype = I
    lib.gqa_kv_append.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
    lib.gqa_decode_workspace_bytes.restype = SZ
    lib.gqa_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.gqa_decode.restype = I
    lib.gqa_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P, SZ, I, P]
    lib.gqa_decode_append.restype = I
    lib.gqa_decode_append.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I, P, SZ, I, P]
    lib.gqa_decode_noalloc.restype = I
    lib.gqa_decode_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, P]
    lib.gqa_decode_paged_workspace_bytes.restype = SZ
    lib.gqa_decode_paged_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.gqa_decode_paged.restype = I
    lib.gqa_decode_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P, SZ, I, P]
    lib.gqa_decode_append_paged.restype = I
    lib.gqa_decode_append_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P, SZ, I, P]
    lib.gqa_kv_append_paged.restype = I
    lib.gqa_kv_append_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P]
    lib.gqa_decode_int8_workspace_bytes.restype = SZ
    lib.gqa_decode_int8_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.gqa_decode_int8.restype = I
    lib.gqa_decode_int8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I, P, SZ, P]
    lib.gqa_kv_append_int8.restype = I
    lib.gqa_kv_append_int8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P]
    lib.gqa_prefill_causal.restype = I
    lib.gqa_prefill_causal.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gqa_prefill_causal_varlen.restype = I
    lib.gqa_prefill_causal_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gqa_kv_project_workspace_bytes.restype = SZ
    lib.gqa_kv_project_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.gqa_kv_project_append.restype = I
    lib.gqa_kv_project_append.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, SZ, I, P]
    lib.gqa_meanpool_kv.restype = I
    lib.gqa_meanpool_kv.argtypes = [P, P, I64, I, I, I64, I, P]
    lib.gqa_get_last_error.restype = I
    lib.gqa_get_last_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.gqa_status_string.restype = ctypes.c_char_p
    lib.gqa_status_string.argtypes = [I]
    return lib


_lib = _load()


def library():
    """The loaded ctypes handle (for tests that call the C ABI directly)."""
    return _lib


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    if t.dtype == torch.float32:
        return GQA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != GQA_OK:
        raise GqaError(fn, status)


def gqa_kv_append(k_cache, v_cache, k_new, v_new, pos, stream=None) -> None:
    """k_cache/v_cache [B,K,S_max,d] (in place), k_new/v_new [B,K,d], pos [B] int32."""
    B, K, S_max, d = k_cache.shape
    assert v_cache.shape == k_cache.shape and k_new.shape == (B, K, d) and v_new.shape == (B, K, d)
    assert pos.dtype == torch.int32 and pos.shape == (B,)
    _check("gqa_kv_append", _lib.gqa_kv_append(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(pos),
                                               B, K, S_max, d, _dtype(k_cache), _stream(stream)))


def gqa_decode_workspace_bytes(B: int, H: int, K: int, S_max: int, d: int, num_splits: int = 0) -> int:
    return int(_lib.gqa_decode_workspace_bytes(B, H, K, S_max, d, num_splits))


def gqa_decode(out, q, k_cache, v_cache, seqlens, scale: float, num_splits: int = 0, workspace=None,
               stream=None) -> None:
    """out/q [B,H,d], k_cache/v_cache [B,K,S_max,d], seqlens [B] int32; workspace a uint8 tensor."""
    B, H, d = q.shape
    _, K, S_max, _ = k_cache.shape
    assert out.shape == q.shape and k_cache.shape[0] == B and k_cache.shape[3] == d
    assert v_cache.shape == k_cache.shape and seqlens.dtype == torch.int32 and seqlens.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_decode", _lib.gqa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, H, K,
                                         S_max, d, float(scale), int(num_splits), _ptr(workspace), ws_bytes,
                                         _dtype(q), _stream(stream)))


def gqa_decode_append(out, q, k_cache, v_cache, k_new, v_new, pos, scale: float, num_splits: int = 0,
                      workspace=None, stream=None) -> None:
    """Append k_new/v_new [B,K,d] at row pos[b], then decode over pos[b] + 1 keys (one pass)."""
    B, H, d = q.shape
    _, K, S_max, _ = k_cache.shape
    assert out.shape == q.shape and k_cache.shape[0] == B and k_cache.shape[3] == d
    assert v_cache.shape == k_cache.shape and k_new.shape == (B, K, d) and v_new.shape == (B, K, d)
    assert pos.dtype == torch.int32 and pos.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_decode_append", _lib.gqa_decode_append(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new),
                                                       _ptr(v_new), _ptr(pos), B, H, K, S_max, d, float(scale),
                                                       int(num_splits), _ptr(workspace), ws_bytes, _dtype(q),
                                                       _stream(stream)))


def gqa_decode_noalloc(out, q, k_cache, v_cache, seqlens, scale: float, num_splits: int = 0, stream=None) -> None:
    """gqa_decode with the library's own static scratch instead of a caller workspace.

    For callers that cannot allocate device memory at decode time. Raises
    GqaError(GQA_ERR_SCRATCH_LIMIT) when the split-KV partials of this shape
    and split count need more than GQA_NOALLOC_SCRATCH_BYTES. Calls that
    overlap on the GPU share the scratch and race.
    """
    B, H, d = q.shape
    _, K, S_max, _ = k_cache.shape
    assert out.shape == q.shape and k_cache.shape[0] == B and k_cache.shape[3] == d
    assert v_cache.shape == k_cache.shape and seqlens.dtype == torch.int32 and seqlens.shape == (B,)
    _check("gqa_decode_noalloc", _lib.gqa_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                                         _ptr(seqlens), B, H, K, S_max, d, float(scale),
                                                         int(num_splits), _dtype(q), _stream(stream)))


def gqa_decode_paged_workspace_bytes(B: int, H: int, K: int, d: int, block_size: int, max_blocks: int,
                                     num_splits: int = 0) -> int:
    return int(_lib.gqa_decode_paged_workspace_bytes(B, H, K, d, block_size, max_blocks, num_splits))


def _paged_shapes(q, k_pool, v_pool, block_table):
    B, H, d = q.shape
    num_blocks, K, block_size, dk = k_pool.shape
    assert dk == d and v_pool.shape == k_pool.shape
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == B
    return B, H, K, d, num_blocks, block_size, block_table.shape[1]


def gqa_decode_paged(out, q, k_pool, v_pool, block_table, seqlens, scale: float, num_splits: int = 0,
                     workspace=None, stream=None) -> None:
    """out/q [B,H,d], pools [num_blocks,K,block_size,d], block_table [B,max_blocks] int32, seqlens [B] int32."""
    B, H, K, d, nb, bs, mb = _paged_shapes(q, k_pool, v_pool, block_table)
    assert out.shape == q.shape and seqlens.dtype == torch.int32 and seqlens.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_decode_paged", _lib.gqa_decode_paged(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                                     _ptr(block_table), _ptr(seqlens), B, H, K, d, nb, bs, mb,
                                                     float(scale), int(num_splits), _ptr(workspace), ws_bytes,
                                                     _dtype(q), _stream(stream)))


def gqa_decode_append_paged(out, q, k_pool, v_pool, k_new, v_new, block_table, pos, scale: float,
                            num_splits: int = 0, workspace=None, stream=None) -> None:
    """Append k_new/v_new [B,K,d] at key pos[b] of the paged cache, then decode over pos[b] + 1 keys."""
    B, H, K, d, nb, bs, mb = _paged_shapes(q, k_pool, v_pool, block_table)
    assert out.shape == q.shape and k_new.shape == (B, K, d) and v_new.shape == (B, K, d)
    assert pos.dtype == torch.int32 and pos.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_decode_append_paged",
           _lib.gqa_decode_append_paged(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(k_new), _ptr(v_new),
                                        _ptr(block_table), _ptr(pos), B, H, K, d, nb, bs, mb, float(scale),
                                        int(num_splits), _ptr(workspace), ws_bytes, _dtype(q), _stream(stream)))


def gqa_kv_append_paged(k_pool, v_pool, k_new, v_new, block_table, pos, stream=None) -> None:
    """pools [num_blocks,K,block_size,d] (in place), k_new/v_new [B,K,d], block_table [B,max_blocks], pos [B]."""
    num_blocks, K, block_size, d = k_pool.shape
    B = k_new.shape[0]
    assert v_pool.shape == k_pool.shape and k_new.shape == (B, K, d) and v_new.shape == (B, K, d)
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == B
    assert pos.dtype == torch.int32 and pos.shape == (B,)
    _check("gqa_kv_append_paged",
           _lib.gqa_kv_append_paged(_ptr(k_pool), _ptr(v_pool), _ptr(k_new), _ptr(v_new), _ptr(block_table),
                                    _ptr(pos), B, K, d, num_blocks, block_size, block_table.shape[1],
                                    _dtype(k_pool), _stream(stream)))


def gqa_decode_int8_workspace_bytes(B: int, H: int, K: int, S_max: int, d: int, num_splits: int = 0) -> int:
    return int(_lib.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, num_splits))


def gqa_decode_int8(out, q, k_codes, k_scales, v_codes, v_scales, seqlens, scale: float, num_splits: int = 0,
                    workspace=None, stream=None) -> None:
    """out/q [B,H,d] bf16; codes [B,K,S_max,d] int8; scales [B,K,S_max] float32; seqlens [B] int32."""
    B, H, d = q.shape
    _, K, S_max, _ = k_codes.shape
    assert out.shape == q.shape and q.dtype == torch.bfloat16 and k_codes.dtype == torch.int8
    assert v_codes.shape == k_codes.shape and v_codes.dtype == torch.int8
    assert k_scales.shape == (B, K, S_max) and v_scales.shape == k_scales.shape and k_scales.dtype == torch.float32
    assert seqlens.dtype == torch.int32 and seqlens.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_decode_int8", _lib.gqa_decode_int8(_ptr(out), _ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                                   _ptr(v_scales), _ptr(seqlens), B, H, K, S_max, d, float(scale),
                                                   int(num_splits), _ptr(workspace), ws_bytes, _stream(stream)))


def gqa_kv_append_int8(k_codes, k_scales, v_codes, v_scales, k_new, v_new, pos, stream=None) -> None:
    """Quantize k_new/v_new [B,K,d] bf16 into the 8-bit caches at key pos[b] (codes and scales in place)."""
    B, K, S_max, d = k_codes.shape
    assert k_new.shape == (B, K, d) and v_new.shape == (B, K, d) and k_new.dtype == torch.bfloat16
    assert pos.dtype == torch.int32 and pos.shape == (B,)
    _check("gqa_kv_append_int8", _lib.gqa_kv_append_int8(_ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                                         _ptr(v_scales), _ptr(k_new), _ptr(v_new), _ptr(pos), B, K,
                                                         S_max, d, _stream(stream)))


def gqa_prefill_causal(out, q, k, v, scale: float, k_cache=None, v_cache=None, stream=None) -> None:
    """out/q [B,S,H,d], k/v [B,S,K,d]; optional caches [B,K,S_max,d] get rows 0..S-1."""
    B, S, H, d = q.shape
    K = k.shape[2]
    assert out.shape == q.shape and k.shape == (B, S, K, d) and v.shape == k.shape
    S_max = k_cache.shape[2] if k_cache is not None else S
    if k_cache is not None:
        assert k_cache.shape == (B, K, S_max, d) and v_cache is not None and v_cache.shape == k_cache.shape
    _check("gqa_prefill_causal", _lib.gqa_prefill_causal(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache),
                                                         _ptr(v_cache), B, S, H, K, S_max, d, float(scale),
                                                         _dtype(q), _stream(stream)))


def gqa_prefill_causal_varlen(out, q, k, v, cu_seqlens, scale: float, k_cache=None, v_cache=None,
                              stream=None) -> None:
    """Packed out/q [T,H,d], k/v [T,K,d], cu_seqlens [B+1] int32; optional caches [B,K,S_max,d]."""
    T, H, d = q.shape
    K = k.shape[1]
    B = cu_seqlens.shape[0] - 1
    assert out.shape == q.shape and k.shape == (T, K, d) and v.shape == k.shape and cu_seqlens.dtype == torch.int32
    S_max = k_cache.shape[2] if k_cache is not None else 0
    if k_cache is not None:
        assert k_cache.shape == (B, K, S_max, d) and v_cache is not None and v_cache.shape == k_cache.shape
    _check("gqa_prefill_causal_varlen",
           _lib.gqa_prefill_causal_varlen(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(cu_seqlens), B, T, H, K, S_max, d, float(scale), _dtype(q),
                                          _stream(stream)))


def gqa_kv_project_workspace_bytes(B: int, T: int, K: int, d: int, d_model: int) -> int:
    return int(_lib.gqa_kv_project_workspace_bytes(B, T, K, d, d_model))


def gqa_kv_project_append(k_cache, v_cache, x, w_kv, pos=None, workspace=None, stream=None) -> None:
    """x [B,T,d_model], w_kv [K,2d,d_model] (bf16); caches [B,K,S_max,d]; pos [B] int32 or None (0)."""
    B, T, d_model = x.shape
    K, two_d, dm = w_kv.shape
    d = two_d // 2
    S_max = k_cache.shape[2]
    assert dm == d_model and k_cache.shape == (B, K, S_max, d) and v_cache.shape == k_cache.shape
    if pos is not None:
        assert pos.dtype == torch.int32 and pos.shape == (B,)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("gqa_kv_project_append",
           _lib.gqa_kv_project_append(_ptr(k_cache), _ptr(v_cache), _ptr(x), _ptr(w_kv), _ptr(pos), B, T, K, S_max,
                                      d, d_model, _ptr(workspace), ws_bytes, _dtype(x), _stream(stream)))


def gqa_meanpool_kv(dst, src, stream=None) -> None:
    """src [outer, H, inner] -> dst [outer, K, inner]."""
    outer, H, inner = src.shape
    K = dst.shape[1]
    assert dst.shape == (outer, K, inner)
    _check("gqa_meanpool_kv", _lib.gqa_meanpool_kv(_ptr(dst), _ptr(src), outer, H, K, inner, _dtype(src),
                                                   _stream(stream)))


def gqa_get_last_error(stream=None) -> Tuple[int, int]:
    """(status, bits): synchronises the stream, reads and clears the device error word."""
    bits = ctypes.c_uint32(0)
    status = _lib.gqa_get_last_error(_stream(stream), ctypes.byref(bits))
    return int(status), int(bits.value)
