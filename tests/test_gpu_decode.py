"""GPU parity of gqa_decode with the float64 oracle.

Small shapes are compared element by element (several tiles, ragged tails,
NaN in every cache row past a sequence's length). The full-size workloads run
in the launch configuration the benchmark times and are compared on sampled
(b, h) rows, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import Guarded, assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    from kv_cache_02_b200 import gqa as g

    return g


def run_decode(gqa, inp, scale, num_splits=0, guarded=True):
    q = dev(inp["q"])
    kc, vc = dev(inp["k_cache"]), dev(inp["v_cache"])
    lens = dev(inp["seqlens"].astype(np.int32))
    B, H, d = inp["q"].shape
    K, S_max = inp["k_cache"].shape[1], inp["k_cache"].shape[2]
    ws_bytes = gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, num_splits)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    out = Guarded((B, H, d), q.dtype)
    gqa.gqa_decode(out.t, q, kc, vc, lens, scale, num_splits, ws if ws_bytes else None)
    status = gqa.gqa_get_last_error()
    assert out.intact(), "write outside the output buffer"
    return host(out.t), status


def make(B, H, K, d, S_max, lens, dtype, seed):
    lens = np.asarray(lens, np.int32)
    return {
        "q": synth.normal((B, H, d), dtype, seed, 1),
        "k_cache": synth.cache(B * K, S_max, d, dtype, seed, 2, lens, K).reshape(B, K, S_max, d),
        "v_cache": synth.cache(B * K, S_max, d, dtype, seed, 3, lens, K).reshape(B, K, S_max, d),
        "seqlens": lens,
    }


SMALL = [
    # B, H, K, d, S_max, lens
    (3, 16, 4, 128, 300, (300, 1, 77)),          # G = 4, ragged, one-row sequence
    (4, 64, 8, 128, 1000, (0, 999, 1000, 513)),   # G = 8, an empty sequence
    (2, 8, 8, 64, 200, (200, 65)),                # G = 1 (MHA), d = 64
    (2, 64, 1, 128, 700, (700, 129)),             # G = 64 (MQA): eight head slices
    (2, 12, 2, 64, 150, (150, 16)),               # G = 6
    (1, 24, 2, 128, 333, (333,)),                 # G = 12: slices of 8 and 4 heads
    (3, 128, 2, 128, 260, (260, 1, 129)),         # G = 64, two KV heads: the tensor-core wide-group path
    (2, 128, 1, 128, 500, (500, 300)),            # G = 128: two slices of 64 heads
]


@pytest.mark.parametrize("num_splits", [0, 1, 3])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: f"B{s[0]}H{s[1]}K{s[2]}d{s[3]}S{s[4]}")
def test_decode_bf16_small(gqa, shape, num_splits):
    B, H, K, d, S_max, lens = shape
    inp = make(B, H, K, d, S_max, lens, synth.BF16, 0xDEC0 + B * 31 + H + K + d)
    scale = 1.0 / np.sqrt(d)
    got, status = run_decode(gqa, inp, scale, num_splits)
    assert status == (0, 0)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale)
    assert_close(got, ref, f"{shape} splits={num_splits}")
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(oracle.widen(got[b]) == 0.0)


@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_decode_f32_tiny_workload(gqa, num_splits):
    w = synth.DECODE_WORKLOADS["tiny_decode_b1_h8_k2_d64_s128_f32"]
    inp = synth.decode_inputs(w)
    scale = 1.0 / np.sqrt(w.d)
    got, status = run_decode(gqa, inp, scale, num_splits)
    assert status == (0, 0)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale)
    assert_close(got, ref, "tiny f32")


@pytest.mark.parametrize("shape", [(3, 64, 2, 128, 200, (200, 0, 31)), (2, 8, 4, 64, 90, (90, 40))])
def test_decode_f32_ragged(gqa, shape):
    B, H, K, d, S_max, lens = shape
    inp = make(B, H, K, d, S_max, lens, synth.F32, 0xF320 + H)
    got, status = run_decode(gqa, inp, 0.1, 2)
    assert status == (0, 0)
    assert_close(got, oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], 0.1), str(shape))


def test_decode_split_counts_agree(gqa):
    inp = make(2, 32, 8, 128, 2048, (2048, 1500), synth.BF16, 0x5A5A)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], 0.088)
    outs = []
    for ns in (1, 2, 7, 32):
        got, status = run_decode(gqa, inp, 0.088, ns)
        assert status == (0, 0)
        assert_close(got, ref, f"splits={ns}")
        outs.append(oracle.widen(got))
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) < 2e-2


def test_decode_bad_length_reported_and_zeroed(gqa):
    inp = make(3, 16, 4, 128, 64, (64, 64, 10), synth.BF16, 0xBAD)
    inp["seqlens"] = np.array([64, 65, 10], np.int32)  # 65 > S_max
    got, (status, bits) = run_decode(gqa, inp, 0.1)
    assert status == gqa.GQA_ERR_DEVICE and bits & gqa.GQA_DEVERR_SEQLEN
    assert np.all(oracle.widen(got[1]) == 0.0)
    ok = np.array([64, 0, 10], np.int32)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], ok, 0.1)
    assert_close(got[[0, 2]], ref[[0, 2]], "valid rows next to a bad one")


# ---------------------------------------------------------------------------
# full-size workloads, launch configuration of the benchmark, sampled rows

FULL = ["llama3_8b_decode_b8_h32_k8_d128_s8192", "ragged_70b_decode_b32_h64_k8_d128_s1k_16k",
        "long_ctx_gqa_b1_h64_k8_d128_s131072", "long_ctx_mqa_b1_h64_k1_d128_s131072"]


@pytest.mark.parametrize("name", FULL)
def test_decode_full_size_sampled(gqa, name):
    w = synth.DECODE_WORKLOADS[name]
    inp = synth.decode_inputs(w)
    if w.append:
        # the benchmark's step: append the new token at pos, then decode over pos + 1 rows
        kc, vc = oracle.kv_append(inp["k_cache"], inp["v_cache"], inp["k_new"], inp["v_new"], inp["pos"])
        tk, tv = dev(inp["k_cache"]), dev(inp["v_cache"])
        gqa.gqa_kv_append(tk, tv, dev(inp["k_new"]), dev(inp["v_new"]), dev(inp["pos"]))
        assert np.array_equal(host(tk), kc) and np.array_equal(host(tv), vc)
        inp["k_cache"], inp["v_cache"] = kc, vc
    scale = 1.0 / np.sqrt(w.d)
    got, status = run_decode(gqa, inp, scale, 0)
    assert status == (0, 0)
    assert np.all(np.isfinite(oracle.widen(got)))
    rng = np.random.default_rng(7)
    sel = np.stack([rng.integers(0, w.B, 48), rng.integers(0, w.H, 48)], 1)
    sel = np.concatenate([sel, [[0, 0], [w.B - 1, w.H - 1]]]).astype(np.int32)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale, sel=sel)
    assert_close(got[sel[:, 0], sel[:, 1]], ref, name)


@pytest.mark.parametrize("name", ["ragged_70b_decode_b32_h64_k8_d128_s1k_16k", "long_ctx_mqa_b1_h64_k1_d128_s131072"])
def test_decode_repeats_bit_for_bit(gqa, name):
    """The persistent CTAs take work items in a different order on every call;
    the result must not depend on that order."""
    w = synth.DECODE_WORKLOADS[name]
    inp = synth.decode_inputs(w)
    q, kc, vc, lens = dev(inp["q"]), dev(inp["k_cache"]), dev(inp["v_cache"]), dev(inp["seqlens"])
    ws_bytes = gqa.gqa_decode_workspace_bytes(w.B, w.H, w.K, w.S_max, w.d, 0)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(4):
        out = torch.full_like(q, float("nan"))
        gqa.gqa_decode(out, q, kc, vc, lens, 1.0 / np.sqrt(w.d), 0, ws)
        assert gqa.gqa_get_last_error() == (0, 0)
        outs.append(host(out))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("name", ["llama3_8b_decode_b8_h32_k8_d128_s8192", "long_ctx_mqa_b1_h64_k1_d128_s131072"])
def test_decode_graph_replay(gqa, name):
    """gqa_decode captured in a CUDA graph and replayed with new queries gives
    the eager call's bits: the persistent kernel's work counter in the
    workspace is left reset by every launch, although a replay repeats it."""
    w = synth.DECODE_WORKLOADS[name]
    inp = synth.decode_inputs(w)
    q, kc, vc, lens = dev(inp["q"]), dev(inp["k_cache"]), dev(inp["v_cache"]), dev(inp["seqlens"])
    ws_bytes = gqa.gqa_decode_workspace_bytes(w.B, w.H, w.K, w.S_max, w.d, 0)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(w.d)
    out, ref = torch.empty_like(q), torch.empty_like(q)
    gqa.gqa_decode(out, q, kc, vc, lens, scale, 0, ws)  # eager first: one-time attribute setup
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gqa.gqa_decode(out, q, kc, vc, lens, scale, 0, ws)
    for rep in range(3):
        q.copy_(dev(synth.normal((w.B, w.H, w.d), synth.BF16, w.seed, 20 + rep)))
        out.fill_(float("nan"))
        g.replay()
        gqa.gqa_decode(ref, q, kc, vc, lens, scale, 0, ws)
        assert gqa.gqa_get_last_error() == (0, 0)
        assert np.array_equal(host(out), host(ref)), f"replay {rep}"
    del g


# ---------------------------------------------------------------------------
# automatic splits: many splits per unit, and the combine of many partials

AUTO = [
    # B, H, K, d, S_max, lens
    (1, 8, 1, 128, 65536, (65536,)),                                  # one unit, a wide combine
    (37, 16, 2, 128, 700, tuple(int(x) for x in np.random.default_rng(3).integers(0, 701, 37))),
    (64, 8, 8, 64, 130, (1, 63, 64, 65, 127, 128, 129, 130) * 8),     # tile-edge lengths, many small units
    (3, 64, 1, 128, 9000, (9000, 4097, 1)),                           # MQA: eight head slices per unit
]


@pytest.mark.parametrize("shape", AUTO, ids=lambda s: f"B{s[0]}H{s[1]}K{s[2]}d{s[3]}S{s[4]}")
def test_decode_auto_splits(gqa, shape):
    B, H, K, d, S_max, lens = shape
    inp = make(B, H, K, d, S_max, lens, synth.BF16, 0x57A0 + B + H)
    scale = 1.0 / np.sqrt(d)
    got, status = run_decode(gqa, inp, scale, 0)
    assert status == (0, 0)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale)
    assert_close(got, ref, str(shape[:5]))


def test_decode_workspace_needs_no_initialisation(gqa):
    inp = make(4, 32, 8, 128, 3000, (3000, 2999, 1, 1500), synth.BF16, 0x57B0)
    B, H, d = inp["q"].shape
    q, kc, vc = dev(inp["q"]), dev(inp["k_cache"]), dev(inp["v_cache"])
    lens = dev(inp["seqlens"])
    ws_bytes = gqa.gqa_decode_workspace_bytes(B, H, 8, 3000, d, 0)
    ref = oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], 0.1)
    for fill in (0xFF, 0x00, 0xA5):
        ws = torch.full((ws_bytes,), fill, dtype=torch.uint8, device="cuda")
        for _ in range(2):  # the same workspace twice in a row
            out = torch.empty_like(q)
            gqa.gqa_decode(out, q, kc, vc, lens, 0.1, 0, ws)
            assert gqa.gqa_get_last_error() == (0, 0)
            assert_close(host(out), ref, f"fill {fill:#x}")


# ---------------------------------------------------------------------------
# gqa_decode_append: the append fused into the decode pass

def run_decode_append(gqa, inp, kn, vn, pos, scale, num_splits=0):
    q = dev(inp["q"])
    kc, vc = dev(inp["k_cache"]), dev(inp["v_cache"])
    B, H, d = inp["q"].shape
    K, S_max = inp["k_cache"].shape[1], inp["k_cache"].shape[2]
    ws_bytes = gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, num_splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = Guarded((B, H, d), q.dtype)
    gqa.gqa_decode_append(out.t, q, kc, vc, dev(kn), dev(vn), dev(np.asarray(pos, np.int32)), scale, num_splits, ws)
    status = gqa.gqa_get_last_error()
    assert out.intact(), "write outside the output buffer"
    return host(out.t), host(kc), host(vc), status


APPEND = [
    # B, H, K, d, S_max, pos, dtype
    (4, 32, 8, 128, 2048, (2047, 1000, 0, 63), synth.BF16),   # token rows at tile edges and at 0
    (3, 64, 1, 128, 700, (699, 64, 129), synth.BF16),          # MQA: head slices share the row
    (2, 16, 2, 64, 300, (299, 17), synth.BF16),
    (2, 8, 2, 64, 128, (127, 5), synth.F32),                   # f32: append launch + decode
]


@pytest.mark.parametrize("num_splits", [0, 1, 5])
@pytest.mark.parametrize("shape", APPEND, ids=lambda s: f"B{s[0]}H{s[1]}K{s[2]}d{s[3]}S{s[4]}{'f32' if s[6] == synth.F32 else ''}")
def test_decode_append_equals_append_then_decode(gqa, shape, num_splits):
    B, H, K, d, S_max, pos, dt = shape
    pos = np.asarray(pos, np.int32)
    inp = make(B, H, K, d, S_max, pos, dt, 0xA99E + H + d)  # rows >= pos are NaN before the append
    kn, vn = synth.normal((B, K, d), dt, 0xA99F, 5), synth.normal((B, K, d), dt, 0xA99F, 6)
    scale = 1.0 / np.sqrt(d)
    got, kc, vc, status = run_decode_append(gqa, inp, kn, vn, pos, scale, num_splits)
    assert status == (0, 0)
    want_k, want_v = oracle.kv_append(inp["k_cache"], inp["v_cache"], kn, vn, pos)
    assert np.array_equal(kc.view(np.uint8), want_k.view(np.uint8)) and np.array_equal(vc.view(np.uint8), want_v.view(np.uint8))
    ref = oracle.decode(inp["q"], want_k, want_v, pos + 1, scale)
    assert_close(got, ref, f"{shape[:5]} splits={num_splits}")


def test_decode_append_bad_position(gqa):
    B, H, K, d, S_max = 3, 16, 4, 128, 64
    pos = np.array([S_max, 10, -1], np.int32)
    inp = make(B, H, K, d, S_max, np.array([S_max, 10, 0], np.int32), synth.BF16, 0xBAD2)
    kn, vn = synth.normal((B, K, d), synth.BF16, 0xBAD3, 5), synth.normal((B, K, d), synth.BF16, 0xBAD3, 6)
    got, kc, vc, (status, bits) = run_decode_append(gqa, inp, kn, vn, pos, 0.1)
    assert status == gqa.GQA_ERR_DEVICE and bits & gqa.GQA_DEVERR_APPEND_POS
    assert np.all(oracle.widen(got[0]) == 0.0) and np.all(oracle.widen(got[2]) == 0.0)
    want_k, want_v = oracle.kv_append(inp["k_cache"], inp["v_cache"], kn, vn, pos)
    assert np.array_equal(kc.view(np.uint8), want_k.view(np.uint8)) and np.array_equal(vc.view(np.uint8), want_v.view(np.uint8))
    ref = oracle.decode(inp["q"], want_k, want_v, np.array([0, 11, 0], np.int32), 0.1)
    assert_close(got[1:2], ref[1:2], "valid row next to bad ones")


def test_decode_append_full_size_sampled(gqa):
    w = synth.DECODE_WORKLOADS["llama3_8b_decode_b8_h32_k8_d128_s8192"]
    inp = synth.decode_inputs(w)
    scale = 1.0 / np.sqrt(w.d)
    got, kc, vc, status = run_decode_append(gqa, inp, inp["k_new"], inp["v_new"], inp["pos"], scale)
    assert status == (0, 0)
    want_k, want_v = oracle.kv_append(inp["k_cache"], inp["v_cache"], inp["k_new"], inp["v_new"], inp["pos"])
    assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v)
    rng = np.random.default_rng(8)
    sel = np.stack([rng.integers(0, w.B, 48), rng.integers(0, w.H, 48)], 1).astype(np.int32)
    ref = oracle.decode(inp["q"], want_k, want_v, inp["pos"] + 1, scale, sel=sel)
    assert_close(got[sel[:, 0], sel[:, 1]], ref, "fused append + decode, Llama-3-8B layer")
