"""GPU parity of the 8-bit KV-cache calls with the float64 oracle.

The decode runs over random int8 codes and per-row scales (rows past each
length hold code -128 and a NaN scale, so a leak poisons the output) and is
compared with the oracle's float64 decode of code * scale. The quantizing
append is compared bit for bit (codes and scales) with the oracle's
quantizer, which decides every code in the same float32 arithmetic.
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


def make8(B, H, K, S_max, lens, seed, d=128):
    lens = np.asarray(lens, np.int32)
    kc, ks = synth.int8_cache(B * K, S_max, d, seed, synth.STREAM_K8, synth.STREAM_KSCALE, lens, K)
    vc, vs = synth.int8_cache(B * K, S_max, d, seed, synth.STREAM_V8, synth.STREAM_VSCALE, lens, K)
    return {"q": synth.normal((B, H, d), synth.BF16, seed, 1), "k_codes": kc.reshape(B, K, S_max, d),
            "k_scale": ks.reshape(B, K, S_max), "v_codes": vc.reshape(B, K, S_max, d),
            "v_scale": vs.reshape(B, K, S_max), "seqlens": lens}


def run_int8(gqa, inp, scale, num_splits):
    B, H, d = inp["q"].shape
    K, S_max = inp["k_codes"].shape[1:3]
    wsb = gqa.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, num_splits)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if wsb else None
    out = Guarded((B, H, d), torch.bfloat16)
    gqa.gqa_decode_int8(out.t, dev(inp["q"]), dev(inp["k_codes"]), dev(inp["k_scale"]), dev(inp["v_codes"]),
                        dev(inp["v_scale"]), dev(inp["seqlens"]), scale, num_splits, ws)
    status = gqa.gqa_get_last_error()
    assert out.intact(), "write outside the output buffer"
    return host(out.t), status


SMALL = [
    # B, H, K, S_max, lens
    (3, 16, 4, 320, (300, 1, 77)),          # G = 4, ragged, one-key sequence
    (4, 64, 8, 1024, (0, 999, 1024, 513)),  # G = 8, an empty sequence
    (2, 8, 8, 192, (192, 65)),              # MHA
    (2, 64, 1, 704, (700, 129)),            # MQA: eight head slices
    (1, 24, 2, 336, (333,)),                # G = 12: slices of 8 and 4 heads
]


@pytest.mark.parametrize("num_splits", [0, 1, 3])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: f"B{s[0]}H{s[1]}K{s[2]}S{s[3]}")
def test_int8_decode_small(gqa, shape, num_splits):
    B, H, K, S_max, lens = shape
    inp = make8(B, H, K, S_max, lens, 0x1808 + B * 31 + H + K)
    scale = 1.0 / np.sqrt(128)
    got, status = run_int8(gqa, inp, scale, num_splits)
    assert status == (0, 0)
    ref = oracle.decode_int8(inp["q"], inp["k_codes"], inp["k_scale"], inp["v_codes"], inp["v_scale"], inp["seqlens"],
                             scale)
    assert_close(got, ref, f"{shape} splits={num_splits}")
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(oracle.widen(got[b]) == 0.0)


def test_int8_decode_scale_edge_cases(gqa):
    # a negative softmax scale, and scales spanning orders of magnitude across keys
    B, H, K, S_max, lens = 2, 16, 4, 256, (256, 100)
    inp = make8(B, H, K, S_max, lens, 0x1809)
    inp["k_scale"] = inp["k_scale"] * np.where(np.arange(S_max) % 3 == 0, 8.0, 0.125).astype(np.float32)
    for scale in (-0.09, 0.3):
        got, status = run_int8(gqa, inp, scale, 0)
        assert status == (0, 0)
        ref = oracle.decode_int8(inp["q"], inp["k_codes"], inp["k_scale"], inp["v_codes"], inp["v_scale"],
                                 inp["seqlens"], scale)
        assert_close(got, ref, f"scale={scale}")


def test_kv_append_int8_bit_exact(gqa):
    B, K, S_max, d = 5, 8, 64, 128
    pos = np.array([0, 17, 63, 64, -1], np.int32)  # the last two are out of range
    kn, vn = synth.normal((B, K, d), synth.BF16, 0x1A, 5), synth.normal((B, K, d), synth.BF16, 0x1A, 6)
    kn[1, 2] = 0  # a zero row: scale 0, codes 0
    kn[2, 0, :] = np.uint16(0x3F80)  # a constant row (1.0): every code 127
    kc, ks = synth.int8_cache(B * K, S_max, d, 0x1A, synth.STREAM_K8, synth.STREAM_KSCALE)
    vc, vs = synth.int8_cache(B * K, S_max, d, 0x1A, synth.STREAM_V8, synth.STREAM_VSCALE)
    kc, ks, vc, vs = kc.reshape(B, K, S_max, d), ks.reshape(B, K, S_max), vc.reshape(B, K, S_max, d), vs.reshape(
        B, K, S_max)
    gk, gks, gv, gvs = dev(kc), dev(ks), dev(vc), dev(vs)
    gqa.gqa_kv_append_int8(gk, gks, gv, gvs, dev(kn), dev(vn), dev(pos))
    st = gqa.gqa_get_last_error()
    assert st[0] == gqa.GQA_ERR_DEVICE and st[1] == gqa.GQA_DEVERR_APPEND_POS
    rk, rks, rv, rvs = oracle.kv_append_int8(kc, ks, vc, vs, kn, vn, pos)
    assert np.array_equal(host(gk), rk) and np.array_equal(host(gv), rv)
    assert np.array_equal(host(gks).view(np.uint32), rks.view(np.uint32))
    assert np.array_equal(host(gvs).view(np.uint32), rvs.view(np.uint32))
    assert (rk[1, 2, 17] == 0).all() and rks[1, 2, 17] == 0 and (rk[2, 0, 63] == 127).all()


def test_int8_append_then_decode(gqa):
    """The serving step on an 8-bit cache: quantize the new token in, then decode over pos + 1 keys."""
    B, H, K, S_max, d = 4, 32, 8, 512, 128
    pos = np.array([511, 0, 200, 333], np.int32)
    inp = make8(B, H, K, S_max, pos, 0x1B)
    kn, vn = synth.normal((B, K, d), synth.BF16, 0x1B, 5), synth.normal((B, K, d), synth.BF16, 0x1B, 6)
    gk, gks, gv, gvs = dev(inp["k_codes"]), dev(inp["k_scale"]), dev(inp["v_codes"]), dev(inp["v_scale"])
    gqa.gqa_kv_append_int8(gk, gks, gv, gvs, dev(kn), dev(vn), dev(pos))
    wsb = gqa.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, 0)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / np.sqrt(d)
    gqa.gqa_decode_int8(out, dev(inp["q"]), gk, gks, gv, gvs, dev(pos + 1), scale, 0, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    rk, rks, rv, rvs = oracle.kv_append_int8(inp["k_codes"], inp["k_scale"], inp["v_codes"], inp["v_scale"], kn, vn,
                                             pos)
    ref = oracle.decode_int8(inp["q"], rk, rks, rv, rvs, pos + 1, scale)
    assert_close(host(out), ref, "append then decode")


def test_int8_bad_length_reported(gqa):
    inp = make8(2, 16, 4, 128, (128, 50), 0x1C)
    inp["seqlens"] = np.array([129, 50], np.int32)
    got, status = run_int8(gqa, inp, 0.1, 0)
    assert status[0] == gqa.GQA_ERR_DEVICE and status[1] & gqa.GQA_DEVERR_SEQLEN


@pytest.mark.parametrize("name", list(synth.INT8_WORKLOADS))
def test_int8_full_size_sampled(gqa, name):
    inp = synth.int8_inputs(name)
    B, H, d = inp["q"].shape
    scale = 1.0 / np.sqrt(d)
    got, status = run_int8(gqa, inp, scale, 0)
    assert status == (0, 0)
    rng = np.random.default_rng(12)
    sel = np.stack([rng.integers(0, B, 24), rng.integers(0, H, 24)], axis=1)
    sel[0], sel[1] = (0, 0), (B - 1, H - 1)
    ref = oracle.decode_int8(inp["q"], inp["k_codes"], inp["k_scale"], inp["v_codes"], inp["v_scale"], inp["seqlens"],
                             scale, sel=sel)
    assert_close(got[sel[:, 0], sel[:, 1]], ref, name)


def test_int8_decode_repeats_bit_for_bit(gqa):
    """The persistent CTAs take work items in a different order on every call;
    which warp sums which keys, and so the result, must not depend on it."""
    inp = synth.int8_inputs("int8_ragged_70b_decode_b32_h64_k8_d128_s1k_16k")
    B, H, d = inp["q"].shape
    K, S_max = inp["k_codes"].shape[1:3]
    t = {k: dev(inp[k]) for k in ("q", "k_codes", "k_scale", "v_codes", "v_scale", "seqlens")}
    wsb = gqa.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, 0)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(4):
        out = torch.full_like(t["q"], float("nan"))
        gqa.gqa_decode_int8(out, t["q"], t["k_codes"], t["k_scale"], t["v_codes"], t["v_scale"], t["seqlens"],
                            1.0 / np.sqrt(d), 0, ws)
        assert gqa.gqa_get_last_error() == (0, 0)
        outs.append(host(out))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_int8_decode_graph_replay(gqa):
    """gqa_decode_int8 captured in a CUDA graph and replayed gives the eager call's bits."""
    inp = synth.int8_inputs("int8_llama3_8b_decode_b8_h32_k8_d128_s8192")
    B, H, d = inp["q"].shape
    K, S_max = inp["k_codes"].shape[1:3]
    t = {k: dev(inp[k]) for k in ("q", "k_codes", "k_scale", "v_codes", "v_scale", "seqlens")}
    wsb = gqa.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, 0)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    out, ref = torch.empty_like(t["q"]), torch.empty_like(t["q"])

    def call(o):
        gqa.gqa_decode_int8(o, t["q"], t["k_codes"], t["k_scale"], t["v_codes"], t["v_scale"], t["seqlens"],
                            1.0 / np.sqrt(d), 0, ws)

    call(out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(out)
    for rep in range(3):
        t["q"].copy_(dev(synth.normal((B, H, d), synth.BF16, 0x1D, 20 + rep)))
        out.fill_(float("nan"))
        g.replay()
        call(ref)
        assert gqa.gqa_get_last_error() == (0, 0)
        assert np.array_equal(host(out), host(ref)), f"replay {rep}"
    del g
