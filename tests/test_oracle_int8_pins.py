"""Pins for the oracle's 8-bit KV cache: the quantizer and the decode over codes.

The reading (the pages name INT8 KV caches, "GQA 完全拆解", section 更进一步的 KV
压缩, but give no scale convention): symmetric codes in [-127, 127], one
float32 scale per cached row, value = code * scale; quantization in float32,
scale = amax / 127, code = x / scale rounded to nearest with ties to even.

The quantizer is pinned by hand-worked rows, the closed-form error bound
|code * scale - x| <= scale / 2 + |x| 2^-24 (one float division), the amax element landing on +-127, zero rows
and sign symmetry. The decode over codes is pinned against torch's float64
scaled_dot_product_attention on the values torch itself dequantizes, and by
two scale identities that hold for any codes. The last test plants mistakes
in copies of the oracle's C source and shows that each one fails a pin.
"""
import os
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def sdpa_decode(q, kc, vc, lens, scale):
    B, H, d = q.shape
    out = np.zeros((B, H, d))
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        qt = torch.from_numpy(q[b][None, :, None, :])
        kt = torch.from_numpy(np.ascontiguousarray(kc[b][None, :, :n, :]))
        vt = torch.from_numpy(np.ascontiguousarray(vc[b][None, :, :n, :]))
        out[b] = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)[0, :, 0, :].numpy()
    return out


# ---------------------------------------------------------------------------
# quantizer checks (each takes an optional oracle library so mutants can be run)

def check_quantize_hand_rows(lib=None):
    # worked by hand: amax 127 -> scale 1; amax 63.5 -> scale 0.5 (both exact in float)
    x = np.array([[127, 63.5, -1, 0.4, 0.6, -126.5], [63.5, 0.25, 0.75, -0.25, 0, -63.5]], np.float32)
    codes, scales = oracle.quantize_int8(x, lib)
    assert scales.tolist() == [1.0, 0.5]
    # 63.5 / 1 ties to 64 (even); -126.5 ties to -126; 0.25 / 0.5 = 0.5 -> 0; 1.5 -> 2; -0.5 -> 0
    assert codes.tolist() == [[127, 64, -1, 0, 1, -126], [127, 0, 2, 0, 0, -127]]


def check_quantize_bounds(lib=None):
    for dt, seed in ((synth.BF16, 1), (synth.F32, 2)):
        x = synth.normal((300, 128), dt, 0x18 + seed, 1)
        codes, scales = oracle.quantize_int8(x, lib)
        xf = oracle.widen(x)
        amax = np.max(np.abs(xf), axis=1)
        assert np.allclose(scales, amax / 127.0, rtol=2e-7, atol=0)
        # |x - code * scale| <= scale / 2, plus the one float rounding of x / scale: |x| * 2^-24
        err = np.abs(codes.astype(np.float64) * scales[:, None] - xf)
        assert np.all(err <= 0.5 * scales[:, None] + np.abs(xf) * 2.0**-23)
        assert np.mean(err <= 0.5 * scales[:, None]) > 0.99
        assert np.all(np.abs(codes) <= 127)
        rows = np.arange(x.shape[0])
        assert np.all(np.abs(codes[rows, np.argmax(np.abs(xf), axis=1)]) == 127)


def check_quantize_zero_and_sign(lib=None):
    x = synth.normal((50, 64), synth.F32, 0x19, 1)
    x[7] = 0.0
    c1, s1 = oracle.quantize_int8(x, lib)
    c2, s2 = oracle.quantize_int8(-x, lib)
    assert s1[7] == 0.0 and np.all(c1[7] == 0)
    assert np.array_equal(s1, s2) and np.array_equal(c1, -c2)


# ---------------------------------------------------------------------------
# decode over codes

SHAPES = [
    # B, H, K, d, S_max, lens
    (2, 8, 2, 16, 20, (20, 7)),
    (1, 6, 1, 8, 9, (9,)),          # MQA
    (3, 4, 4, 8, 12, (12, 1, 0)),   # MHA, one-key and empty sequences
]


def make8(B, H, K, d, S, lens, seed):
    q = synth.normal((B, H, d), synth.F64, seed, 1)
    kc, ks = synth.int8_cache(B * K, S, d, seed, synth.STREAM_K8, synth.STREAM_KSCALE, np.array(lens), K)
    vc, vs = synth.int8_cache(B * K, S, d, seed, synth.STREAM_V8, synth.STREAM_VSCALE, np.array(lens), K)
    return q, kc.reshape(B, K, S, d), ks.reshape(B, K, S), vc.reshape(B, K, S, d), vs.reshape(B, K, S)


def check_decode_int8_vs_sdpa(lib=None):
    for i, (B, H, K, d, S, lens) in enumerate(SHAPES):
        q, kc, ks, vc, vs = make8(B, H, K, d, S, lens, 0x88 + i)
        lens = np.array(lens, np.int32)
        # torch's own dequantization, rows past each length never used
        kd = torch.from_numpy(kc.astype(np.float64)) * torch.from_numpy(np.nan_to_num(ks).astype(np.float64))[..., None]
        vd = torch.from_numpy(vc.astype(np.float64)) * torch.from_numpy(np.nan_to_num(vs).astype(np.float64))[..., None]
        scale = 1.0 / np.sqrt(d)
        got = oracle.decode_int8(q, kc, ks, vc, vs, lens, scale, lib=lib)
        want = sdpa_decode(q, kd.numpy(), vd.numpy(), lens, scale)
        assert np.all(np.isfinite(got)) and np.max(np.abs(got - want)) <= 1e-12


def check_decode_int8_scale_identities(lib=None):
    B, H, K, d, S, lens = 2, 8, 2, 16, 24, (24, 11)
    q, kc, ks, vc, vs = make8(B, H, K, d, S, lens, 0x99)
    lens = np.array(lens, np.int32)
    base = oracle.decode_int8(q, kc, ks, vc, vs, lens, 0.2, lib=lib)
    # every K scale times 4 == softmax scale times 4 (powers of two keep it exact)
    a = oracle.decode_int8(q, kc, ks * 4, vc, vs, lens, 0.2, lib=lib)
    b = oracle.decode_int8(q, kc, ks, vc, vs, lens, 0.8, lib=lib)
    assert np.max(np.abs(a - b)) <= 1e-12
    # every V scale times 8 == the output times 8
    c = oracle.decode_int8(q, kc, ks, vc, vs * 8, lens, 0.2, lib=lib)
    assert np.max(np.abs(c - 8 * base)) <= 1e-12
    # doubling one key's codes' scale changes the result (the scale is per row, not per tensor)
    ks2 = ks.copy()
    ks2[0, 0, 3] *= 2
    assert np.max(np.abs(oracle.decode_int8(q, kc, ks2, vc, vs, lens, 0.2, lib=lib)[0] - base[0])) > 1e-6


ALL_CHECKS = [check_quantize_hand_rows, check_quantize_bounds, check_quantize_zero_and_sign,
              check_decode_int8_vs_sdpa, check_decode_int8_scale_identities]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_int8_pin(check):
    check()


def test_kv_append_int8_writes_the_quantized_row():
    B, K, d, S = 3, 2, 16, 10
    kc, ks = synth.int8_cache(B * K, S, d, 5, synth.STREAM_K8, synth.STREAM_KSCALE)
    vc, vs = synth.int8_cache(B * K, S, d, 5, synth.STREAM_V8, synth.STREAM_VSCALE)
    kc, ks, vc, vs = kc.reshape(B, K, S, d), ks.reshape(B, K, S), vc.reshape(B, K, S, d), vs.reshape(B, K, S)
    kn, vn = synth.normal((B, K, d), synth.BF16, 5, 5), synth.normal((B, K, d), synth.BF16, 5, 6)
    pos = np.array([0, 9, 10], np.int32)  # the last one is out of range: nothing written
    k2, ks2, v2, vs2 = oracle.kv_append_int8(kc, ks, vc, vs, kn, vn, pos)
    qk, qks = oracle.quantize_int8(kn)
    for b in range(2):
        assert np.array_equal(k2[b, :, pos[b]], qk[b]) and np.array_equal(ks2[b, :, pos[b]], qks[b])
    mask = np.ones((B, K, S), bool)
    mask[0, :, 0] = mask[1, :, 9] = False
    assert np.array_equal(k2[mask], kc[mask]) and np.array_equal(ks2[mask], ks[mask])
    assert np.array_equal(v2[2], vc[2])


# ---------------------------------------------------------------------------
# planted mistakes in the oracle's 8-bit code

MUTANTS = {
    "ties_away_from_zero": ("nearbyintf((float)widen(x, dtype, r * n + i) / sc)",
                            "roundf((float)widen(x, dtype, r * n + i) / sc)"),
    "divides_by_128": ("float sc = amax / 127.0f;", "float sc = amax / 128.0f;"),
    "no_absolute_value": ("float a = fabsf((float)widen(x, dtype, r * n + i));",
                          "float a = (float)widen(x, dtype, r * n + i);"),
    "scale_not_applied": ("(double)((const int8_t*)c->base)[i] * (double)c->scales[i / c->d]",
                          "(double)((const int8_t*)c->base)[i] * 1.0"),
    "scale_per_element": ("(double)c->scales[i / c->d]", "(double)c->scales[i % c->d]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_int8_mistake_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gqa_ref.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    (tmp_path / "m.c").write_text(src.replace(old, new))
    so = str(tmp_path / "m.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread", "-o", so,
                           str(tmp_path / "m.c"), "-lm"])
    lib = oracle.load_library(so)
    failed = []
    for check in ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(lib)
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"
