"""The C ABI on the host: the library loads, exports every symbol that
include/gqa.h declares, and rejects bad arguments before touching the GPU.
Also checks that the oracle and the CUDA path share no code."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_02_b200 import build

    build.build()
    from kv_cache_02_b200 import gqa

    return gqa.library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_symbols() == sorted(["gqa_kv_append", "gqa_decode_workspace_bytes", "gqa_decode",
                                         "gqa_decode_append", "gqa_decode_noalloc",
                                         "gqa_decode_paged_workspace_bytes", "gqa_decode_paged",
                                         "gqa_decode_append_paged", "gqa_kv_append_paged",
                                         "gqa_decode_int8_workspace_bytes", "gqa_decode_int8", "gqa_kv_append_int8",
                                         "gqa_prefill_causal_varlen", "gqa_kv_project_workspace_bytes",
                                         "gqa_kv_project_append",
                                         "gqa_prefill_causal",
                                         "gqa_meanpool_kv", "gqa_get_last_error", "gqa_status_string"])


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_names_match_the_c_abi():
    from kv_cache_02_b200 import gqa

    for name in declared_symbols():
        if name == "gqa_status_string":
            continue
        assert callable(getattr(gqa, name)), name


def test_status_strings(lib):
    assert lib.gqa_status_string(0) == b"GQA_OK"
    assert lib.gqa_status_string(-2) == b"GQA_ERR_SHAPE"
    assert lib.gqa_status_string(-99) == b"GQA_ERR_UNKNOWN"


P = 0x10000  # a fake, 16-byte-aligned device address: never dereferenced by these calls


def test_decode_rejects_bad_arguments(lib):
    f = lib.gqa_decode
    # H % K != 0
    assert f(P, P, P, P, P, 1, 6, 4, 16, 64, 1.0, 0, None, 0, 1, None) == -2
    # unsupported head dim
    assert f(P, P, P, P, P, 1, 8, 2, 16, 96, 1.0, 0, None, 0, 1, None) == -2
    # bad dtype
    assert f(P, P, P, P, P, 1, 8, 2, 16, 64, 1.0, 0, None, 0, 7, None) == -1
    # negative split count
    assert f(P, P, P, P, P, 1, 8, 2, 16, 64, 1.0, -1, None, 0, 1, None) == -1
    # NULL pointer
    assert f(None, P, P, P, P, 1, 8, 2, 16, 64, 1.0, 0, None, 0, 1, None) == -1
    # misaligned pointer
    assert f(P + 2, P, P, P, P, 1, 8, 2, 16, 64, 1.0, 0, None, 0, 1, None) == -3
    # empty batch is a no-op
    assert f(None, None, None, None, None, 0, 8, 2, 16, 64, 1.0, 0, None, 0, 1, None) == 0
    # TMA row coordinates are int32: B*K*S_max must stay below 2^31
    assert f(P, P, P, P, P, 1 << 12, 8, 8, 1 << 16, 128, 1.0, 0, None, 0, 1, None) == -2


def test_append_and_meanpool_reject_bad_arguments(lib):
    assert lib.gqa_kv_append(P, P, P, P, P, 2, 2, 8, 72, 1, None) == -2
    assert lib.gqa_kv_append(P, P, P + 8, P, P, 2, 2, 8, 64, 1, None) == -3
    assert lib.gqa_kv_append(None, P, P, P, P, 2, 2, 8, 64, 1, None) == -1
    assert lib.gqa_kv_append(None, None, None, None, None, 0, 2, 8, 64, 1, None) == 0
    assert lib.gqa_meanpool_kv(P, P, 1, 6, 4, 64, 1, None) == -2
    assert lib.gqa_meanpool_kv(P, P, -1, 8, 4, 64, 1, None) == -1
    assert lib.gqa_meanpool_kv(None, None, 0, 8, 4, 64, 1, None) == 0


def test_paged_calls_reject_bad_arguments(lib):
    f = lib.gqa_decode_paged
    # out, q, k_pool, v_pool, table, seqlens, B, H, K, d, num_blocks, block_size, max_blocks, scale, splits, ws, ws_bytes,
    # dtype, stream
    assert f(P, P, P, P, P, P, 2, 8, 2, 64, 64, 24, 8, 1.0, 0, None, 0, 1, None) == -2     # block size not 16k
    assert f(P, P, P, P, P, P, 2, 8, 2, 64, 64, 0, 8, 1.0, 0, None, 0, 1, None) == -2
    assert f(P, P, P, P, P, P, 2, 8, 2, 64, 64, 16, 0, 1.0, 0, None, 0, 1, None) == -2      # no table columns
    assert f(P, P, P, P, P, P, 2, 6, 4, 64, 64, 16, 8, 1.0, 0, None, 0, 1, None) == -2      # H % K != 0
    assert f(P, P, P, P, P, P, 2, 8, 2, 64, 64, 16, 8, 1.0, 0, None, 0, 0, None) == -6      # f32
    assert f(P, P, P, P, None, P, 2, 8, 2, 64, 64, 16, 8, 1.0, 0, None, 0, 1, None) == -1   # no table
    assert f(P, P, P + 4, P, P, P, 2, 8, 2, 64, 64, 16, 8, 1.0, 0, None, 0, 1, None) == -3  # misaligned pool
    # pool rows num_blocks * K * block_size are TMA row coordinates: below 2^31
    assert f(P, P, P, P, P, P, 2, 8, 8, 64, 1 << 20, 256, 8, 1.0, 0, None, 0, 1, None) == -2
    # a split plan needs a workspace
    assert f(P, P, P, P, P, P, 1, 8, 2, 64, 2048, 16, 2048, 1.0, 0, None, 0, 1, None) == -1
    assert f(None, None, None, None, None, None, 0, 8, 2, 64, 64, 16, 8, 1.0, 0, None, 0, 1, None) == 0
    fa = lib.gqa_decode_append_paged
    assert fa(P, P, P, P, P, P, P, P, 2, 8, 2, 64, 64, 40, 8, 1.0, 0, None, 0, 1, None) == -2
    assert fa(P, P, P, P, None, P, P, P, 2, 8, 2, 64, 64, 16, 8, 1.0, 0, None, 0, 1, None) == -1  # no k_new
    ap = lib.gqa_kv_append_paged
    # k_pool, v_pool, k_new, v_new, table, pos, B, K, d, num_blocks, block_size, max_blocks, dtype, stream
    assert ap(P, P, P, P, P, P, 2, 2, 64, 64, 8, 8, 1, None) == -2      # block size not 16k
    assert ap(P, P, P, P, None, P, 2, 2, 64, 64, 16, 8, 1, None) == -1  # no table
    assert ap(P, P, P, P, P, P, 2, 2, 72, 64, 16, 8, 1, None) == -2     # head dim
    assert ap(None, None, None, None, None, None, 0, 2, 64, 64, 16, 8, 1, None) == 0
    ws = lib.gqa_decode_paged_workspace_bytes
    assert ws(1, 8, 2, 64, 24, 8, 0) == 0 and ws(1, 6, 4, 64, 16, 8, 0) == 0
    assert ws(1, 64, 8, 128, 16, 8192, 0) > 0  # a long sequence is split


def test_int8_calls_reject_bad_arguments(lib):
    f = lib.gqa_decode_int8
    # out, q, k_codes, k_scales, v_codes, v_scales, seqlens, B, H, K, S_max, d, scale, splits, ws, ws_bytes, stream
    assert f(P, P, P, P, P, P, P, 2, 8, 2, 64, 64, 1.0, 0, None, 0, None) == -6     # head dim 64
    assert f(P, P, P, P, P, P, P, 2, 8, 2, 66, 128, 1.0, 0, None, 0, None) == -2    # S_max not a multiple of 4
    assert f(P, P, P, P, P, P, P, 2, 6, 4, 64, 128, 1.0, 0, None, 0, None) == -2    # H % K != 0
    assert f(P, P, P, None, P, P, P, 2, 8, 2, 64, 128, 1.0, 0, None, 0, None) == -1  # no scales
    assert f(P, P, P, P + 4, P, P, P, 2, 8, 2, 64, 128, 1.0, 0, None, 0, None) == -3  # misaligned scales
    assert f(P, P, P, P, P, P, P, 1, 8, 2, 1 << 14, 128, 1.0, 0, None, 0, None) == -1  # split plan, no workspace
    assert f(None, None, None, P, None, P, None, 0, 8, 2, 64, 128, 1.0, 0, None, 0, None) == 0
    a = lib.gqa_kv_append_int8
    assert a(P, P, P, P, P, P, P, 2, 2, 64, 64, None) == -6
    assert a(P, None, P, P, P, P, P, 2, 2, 64, 128, None) == -1
    assert a(None, None, None, None, None, None, None, 0, 2, 64, 128, None) == 0
    ws = lib.gqa_decode_int8_workspace_bytes
    assert ws(1, 8, 2, 64, 64, 0) == 0 and ws(1, 8, 2, 66, 128, 0) == 0
    assert ws(1, 64, 8, 131072, 128, 0) > 0


def test_varlen_prefill_rejects_bad_arguments(lib):
    f = lib.gqa_prefill_causal_varlen
    # out, q, k, v, k_cache, v_cache, cu, B, T, H, K, S_max, d, scale, dtype, stream
    assert f(P, P, P, P, None, None, P, 2, 100, 6, 4, 0, 128, 1.0, 1, None) == -2     # H % K != 0
    assert f(P, P, P, P, None, None, P, 2, 100, 8, 4, 0, 96, 1.0, 1, None) == -2      # head dim
    assert f(P, P, P, P, None, None, P, 2, 100, 8, 4, 0, 128, 1.0, 0, None) == -6     # f32
    assert f(P, P, P, P, P, None, P, 2, 100, 8, 4, 64, 128, 1.0, 1, None) == -1       # one cache pointer
    assert f(P, P, P, P, None, None, None, 2, 100, 8, 4, 0, 128, 1.0, 1, None) == -1  # no cu_seqlens
    assert f(P, P + 8, P, P, None, None, P, 2, 100, 8, 4, 0, 128, 1.0, 1, None) == -3
    assert f(None, None, None, None, None, None, None, 2, 0, 8, 4, 0, 128, 1.0, 1, None) == 0


def test_projection_rejects_bad_arguments(lib):
    f = lib.gqa_kv_project_append
    # k_cache, v_cache, x, w, pos, B, T, K, S_max, d, d_model, ws, ws_bytes, dtype, stream
    assert f(P, P, P, P, None, 2, 1, 8, 64, 96, 4096, None, 0, 1, None) == -2    # head dim
    assert f(P, P, P, P, None, 2, 1, 8, 64, 128, 4000, None, 0, 1, None) == -2   # d_model not a multiple of 64
    assert f(P, P, P, P, None, 2, 1, 8, 64, 128, 4096, None, 0, 0, None) == -6   # f32
    # a 256-token prompt: its d_model is split over CTAs, which needs a workspace
    assert f(P, P, P, P, None, 2, 128, 8, 1024, 128, 4096, None, 0, 1, None) == -1
    assert f(P, P, P + 2, P, None, 2, 1, 8, 64, 128, 4096, None, 0, 1, None) == -3
    assert f(None, None, None, None, None, 0, 1, 8, 64, 128, 4096, None, 0, 1, None) == 0
    ws = lib.gqa_kv_project_workspace_bytes
    assert ws(8, 1, 8, 128, 4096) == 0       # a decode step (<= 16 tokens): the GEMV, no split
    assert ws(2, 128, 8, 128, 4096) > 0      # a short prompt split over d_model
    assert ws(4, 4096, 8, 128, 4096) == 0 and ws(8, 1, 8, 128, 100) == 0


def test_prefill_rejects_bad_arguments(lib):
    f = lib.gqa_prefill_causal
    assert f(P, P, P, P, None, None, 1, 16, 6, 4, 16, 128, 1.0, 1, None) == -2
    assert f(P, P, P, P, P, None, 1, 16, 8, 4, 16, 128, 1.0, 1, None) == -1   # one cache pointer only
    assert f(P, P, P, P, P, P, 1, 32, 8, 4, 16, 128, 1.0, 1, None) == -2      # S > S_max
    assert f(P, P, P, P, None, None, 1, 16, 8, 4, 16, 128, 1.0, 0, None) == -6  # f32 prefill
    assert f(None, None, None, None, None, None, 0, 16, 8, 4, 16, 128, 1.0, 1, None) == 0


def test_workspace_size_is_zero_for_invalid_shapes(lib):
    assert lib.gqa_decode_workspace_bytes(1, 6, 4, 16, 64, 0) == 0
    assert lib.gqa_decode_workspace_bytes(1, 8, 2, 16, 80, 0) == 0
    # long single sequence: the key axis is split, partials need room
    assert lib.gqa_decode_workspace_bytes(1, 64, 8, 131072, 128, 0) > 0


def test_split_planner_choices(lib):
    # The automatic split count, seen through the workspace each plan needs
    # (the partials of nsplit splits): a paged cache gets splits of at least
    # 448 keys (the Llama-3-8B layer: 19 splits of 448 keys, as asked for
    # explicitly of the contiguous cache, not the contiguous cache's 26 of
    # 320), the 8-bit cache about six work items per SM (14 splits), and an
    # explicit split count gives both layouts the same plan.
    B, H, K, d, S = 8, 32, 8, 128, 8192
    contiguous_auto = lib.gqa_decode_workspace_bytes(B, H, K, S, d, 0)
    assert contiguous_auto == lib.gqa_decode_workspace_bytes(B, H, K, S, d, 26)
    paged_auto = lib.gqa_decode_paged_workspace_bytes(B, H, K, d, 16, S // 16, 0)
    assert paged_auto == lib.gqa_decode_workspace_bytes(B, H, K, S, d, 19) < contiguous_auto
    for ns in (1, 3, 19):
        assert lib.gqa_decode_paged_workspace_bytes(B, H, K, d, 16, S // 16, ns) == \
            lib.gqa_decode_workspace_bytes(B, H, K, S, d, ns)
    assert lib.gqa_decode_int8_workspace_bytes(B, H, K, S, d, 0) == lib.gqa_decode_int8_workspace_bytes(B, H, K, S, d, 14)


def _python_imports(path):
    out = set()
    for line in open(path, encoding="utf-8"):
        m = re.match(r"\s*(?:from|import)\s+([\w\.]+)", line)
        if m:
            out.add(m.group(1).split(".")[0])
    return out


def test_oracle_and_cuda_path_share_no_code():
    pkg = os.path.join(ROOT, "kv_cache_02_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            p = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert "oracle" not in _python_imports(p), p
            if f.endswith((".cu", ".cuh", ".h", ".c")):
                assert "oracle" not in open(p, encoding="utf-8").read().lower(), p
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        p = os.path.join(ROOT, "oracle", f)
        if f.endswith(".py"):
            assert "kv_cache_02_b200" not in _python_imports(p), p
        if f.endswith(".c"):
            assert "#include \"" not in open(p, encoding="utf-8").read(), p


def test_binding_refuses_host_tensors(lib):
    """There is no CPU path: the binding raises on host tensors instead of computing anything."""
    import torch

    from kv_cache_02_b200 import gqa

    B, H, K, S, d = 2, 8, 2, 64, 64
    q = torch.zeros((B, H, d), dtype=torch.bfloat16)
    kc = torch.zeros((B, K, S, d), dtype=torch.bfloat16)
    lens = torch.full((B,), S, dtype=torch.int32)
    calls = [
        lambda: gqa.gqa_decode(torch.empty_like(q), q, kc, kc, lens, 0.125),
        lambda: gqa.gqa_decode_append(torch.empty_like(q), q, kc, kc, kc[:, :, 0], kc[:, :, 0], lens, 0.125),
        lambda: gqa.gqa_kv_append(kc, kc, kc[:, :, 0], kc[:, :, 0], lens),
        lambda: gqa.gqa_meanpool_kv(torch.empty((1, K, 16), dtype=torch.bfloat16),
                                    torch.zeros((1, H, 16), dtype=torch.bfloat16)),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="on the GPU"):
            call()
