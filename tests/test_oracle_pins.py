"""Pins for the float64 oracle: what the pages and the mathematics fix.

Nothing here compares the oracle with itself. Each check ties it to a number
the pages print, a closed form, a special case that reduces to an independent
library routine (torch's float64 CPU scaled_dot_product_attention, which takes
grouped K/V heads directly), or brute force on tiny inputs. The last test
plants mistakes in copies of the oracle's C source and shows that every one of
them fails at least one pin.
"""
import os
import re
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, stream=1):
    return synth.normal(shape, synth.F64, seed, stream)


def sdpa_decode(q, kc, vc, lens, scale):
    """Library cross-check: one query row per head against the first lens[b] keys."""
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
# pin checks; each takes an optional oracle library so mutants can be run

DECODE_SHAPES = [
    # B, H, K, d, S_max, lens
    (2, 8, 2, 16, 9, (9, 5)),
    (1, 4, 4, 8, 6, (6,)),          # K = H: MHA
    (2, 6, 1, 8, 7, (7, 3)),        # K = 1: MQA
    (3, 12, 3, 32, 20, (20, 1, 13)),
]


def check_decode_vs_sdpa(lib=None):
    for i, (B, H, K, d, S, lens) in enumerate(DECODE_SHAPES):
        q, kc, vc = rnd((B, H, d), 10 + i, 1), rnd((B, K, S, d), 10 + i, 2), rnd((B, K, S, d), 10 + i, 3)
        scale = 1.0 / np.sqrt(d)
        got = oracle.decode(q, kc, vc, np.array(lens), scale, lib=lib)
        want = sdpa_decode(q, kc, vc, lens, scale)
        assert np.max(np.abs(got - want)) < 1e-12, (B, H, K, d, S, lens)


def check_decode_repeat_kv(lib=None):
    # the Transformers route on the GQA page: repeat each KV head H/K times, then plain MHA
    B, H, K, d, S = 2, 8, 2, 16, 11
    q, kc, vc = rnd((B, H, d), 21, 1), rnd((B, K, S, d), 21, 2), rnd((B, K, S, d), 21, 3)
    lens = np.array([S, S])
    kr = torch.from_numpy(kc).repeat_interleave(H // K, dim=1)
    vr = torch.from_numpy(vc).repeat_interleave(H // K, dim=1)
    want = F.scaled_dot_product_attention(torch.from_numpy(q)[:, :, None, :], kr, vr, scale=0.3)[:, :, 0, :]
    got = oracle.decode(q, kc, vc, lens, 0.3, lib=lib)
    assert np.max(np.abs(got - want.numpy())) < 1e-12


def check_decode_mqa_einsum(lib=None):
    # MQA written as on the GQA page's MQA section: K, V lose the head index ([b, n, d_k])
    B, H, d, n = 2, 6, 8, 10
    q, kk, vv = rnd((B, H, d), 31, 1), rnd((B, n, d), 31, 2), rnd((B, n, d), 31, 3)
    logits = np.einsum("bhk,bnk->bhn", q, kk) * 0.5
    w = np.exp(logits - logits.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    want = np.einsum("bhn,bnv->bhv", w, vv)
    got = oracle.decode(q, kk[:, None], vv[:, None], np.array([n, n]), 0.5, lib=lib)
    assert np.max(np.abs(got - want)) < 1e-12


def check_decode_mha_per_head(lib=None):
    # K = H is standard MHA: every head attends to its own K, V (brute force per head)
    B, H, d, n = 1, 3, 4, 5
    q, kc, vc = rnd((B, H, d), 41, 1), rnd((B, H, n, d), 41, 2), rnd((B, H, n, d), 41, 3)
    got = oracle.decode(q, kc, vc, np.array([n]), 0.7, lib=lib)
    for h in range(H):
        s = [0.7 * sum(q[0, h, i] * kc[0, h, t, i] for i in range(d)) for t in range(n)]
        m = max(s)
        w = [np.exp(x - m) for x in s]
        z = sum(w)
        want = [sum(w[t] * vc[0, h, t, i] for t in range(n)) / z for i in range(d)]
        assert np.max(np.abs(got[0, h] - np.array(want))) < 1e-13


def check_head_mapping_contiguous(lib=None):
    # V of KV head g is the constant g + 1: head h must return h // (H/K) + 1
    B, H, K, d, S = 1, 12, 3, 8, 4
    q, kc = rnd((B, H, d), 51, 1), rnd((B, K, S, d), 51, 2)
    vc = np.zeros((B, K, S, d))
    for g in range(K):
        vc[:, g] = g + 1
    got = oracle.decode(q, kc, vc, np.array([S]), 0.4, lib=lib)
    want = np.repeat((np.arange(H) // (H // K) + 1.0)[:, None], d, axis=1)
    assert np.max(np.abs(got[0] - want)) < 1e-12


def check_identical_keys_mean_of_v(lib=None):
    B, H, K, d, S = 2, 4, 2, 8, 7
    q = rnd((B, H, d), 61, 1)
    kc = np.broadcast_to(rnd((B, K, 1, d), 61, 2), (B, K, S, d)).copy()
    vc = rnd((B, K, S, d), 61, 3)
    lens = np.array([7, 3])
    got = oracle.decode(q, kc, vc, lens, 0.9, lib=lib)
    for b in range(B):
        for h in range(H):
            want = vc[b, h // 2, : lens[b]].mean(0)
            assert np.max(np.abs(got[b, h] - want)) < 1e-14


def check_len1_and_len0(lib=None):
    B, H, K, d, S = 3, 4, 2, 8, 5
    q, kc, vc = rnd((B, H, d), 71, 1), rnd((B, K, S, d), 71, 2), rnd((B, K, S, d), 71, 3)
    got = oracle.decode(q, kc, vc, np.array([1, 0, 1]), 0.5, lib=lib)
    for h in range(H):
        assert np.array_equal(got[0, h], vc[0, h // 2, 0])
        assert np.array_equal(got[2, h], vc[2, h // 2, 0])
    assert np.array_equal(got[1], np.zeros((H, d)))


def check_scale_limits(lib=None):
    B, H, K, d, S = 1, 4, 2, 8, 6
    q, kc, vc = rnd((B, H, d), 81, 1), rnd((B, K, S, d), 81, 2), rnd((B, K, S, d), 81, 3)
    # scale 0: uniform weights
    got = oracle.decode(q, kc, vc, np.array([S]), 0.0, lib=lib)
    for h in range(H):
        assert np.max(np.abs(got[0, h] - vc[0, h // 2].mean(0))) < 1e-14
    # very large scale: the softmax becomes a hard max over the scores
    got = oracle.decode(q, kc, vc, np.array([S]), 1e6, lib=lib)
    for h in range(H):
        t = int(np.argmax(kc[0, h // 2] @ q[0, h]))
        assert np.max(np.abs(got[0, h] - vc[0, h // 2, t])) < 1e-12


def check_shift_and_permutation(lib=None):
    B, H, K, d, S = 1, 6, 2, 8, 9
    q, kc, vc = rnd((B, H, d), 91, 1), rnd((B, K, S, d), 91, 2), rnd((B, K, S, d), 91, 3)
    base = oracle.decode(q, kc, vc, np.array([S]), 0.35, lib=lib)
    # adding one vector to every key shifts each head's scores by a constant
    u = rnd((d,), 91, 4)
    shifted = oracle.decode(q, kc + u, vc, np.array([S]), 0.35, lib=lib)
    assert np.max(np.abs(shifted - base)) < 1e-12
    # permuting key positions together with their values changes nothing
    p = np.random.default_rng(0).permutation(S)
    perm = oracle.decode(q, kc[:, :, p], vc[:, :, p], np.array([S]), 0.35, lib=lib)
    assert np.max(np.abs(perm - base)) < 1e-13


def check_prefill_vs_sdpa(lib=None):
    for i, (B, S, H, K, d) in enumerate([(2, 9, 8, 2, 16), (1, 7, 4, 1, 8), (1, 6, 3, 3, 8)]):
        q, k, v = rnd((B, S, H, d), 101 + i, 1), rnd((B, S, K, d), 101 + i, 2), rnd((B, S, K, d), 101 + i, 3)
        got = oracle.prefill_causal(q, k, v, 0.3, lib=lib)
        tq = torch.from_numpy(q).transpose(1, 2)
        tk = torch.from_numpy(k).transpose(1, 2)
        tv = torch.from_numpy(v).transpose(1, 2)
        want = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.3, enable_gqa=True)
        assert np.max(np.abs(got - want.transpose(1, 2).numpy())) < 1e-12


def check_prefill_rows(lib=None):
    B, S, H, K, d = 2, 8, 4, 2, 8
    q, k, v = rnd((B, S, H, d), 111, 1), rnd((B, S, K, d), 111, 2), rnd((B, S, K, d), 111, 3)
    got = oracle.prefill_causal(q, k, v, 0.5, lib=lib)
    # row 0 sees only key 0: its output is v_0 exactly
    for b in range(B):
        for h in range(H):
            assert np.array_equal(got[b, 0, h], v[b, 0, h // 2])
    # row i is a decode step over a cache holding keys 0..i
    kc, vc = np.transpose(k, (0, 2, 1, 3)).copy(), np.transpose(v, (0, 2, 1, 3)).copy()
    for i in range(S):
        dec = oracle.decode(q[:, i], kc, vc, np.array([i + 1] * B), 0.5, lib=lib)
        assert np.max(np.abs(dec - got[:, i])) < 1e-13
    # changing keys/values after row i leaves rows <= i unchanged
    k2, v2 = k.copy(), v.copy()
    k2[:, 5:] += 3.0
    v2[:, 5:] -= 2.0
    got2 = oracle.prefill_causal(q, k2, v2, 0.5, lib=lib)
    assert np.array_equal(got2[:, :5], got[:, :5])
    assert not np.allclose(got2[:, 5:], got[:, 5:])


def check_meanpool(lib=None):
    # integer-valued heads: the mean is exact in float64
    outer, H, K, inner = 3, 8, 2, 5
    src = np.random.default_rng(1).integers(-50, 50, size=(outer, H, inner)).astype(np.float64)
    got = oracle.meanpool_kv(src, K, lib=lib)
    G = H // K
    for g in range(K):
        # 1-based group g+1 holds heads g*G+1 .. (g+1)*G (the GQA page's range formula)
        heads = [h - 1 for h in range((g * H) // K + 1, ((g + 1) * H) // K + 1)]
        assert np.array_equal(got[:, g], src[:, heads].mean(1))
    # library cross-check on random data, and linearity in the projection sense
    W = rnd((1, 12, 6 * 4), 121, 1)  # [1, H, d_k * d_model]
    got = oracle.meanpool_kv(W, 3, lib=lib)
    want = torch.from_numpy(W).view(1, 3, 4, 24).mean(2).numpy()
    assert np.max(np.abs(got - want)) < 1e-15
    x = rnd((4,), 121, 2)
    Wp = W.reshape(12, 6, 4)
    for g in range(3):
        lhs = got.reshape(3, 6, 4)[g] @ x
        rhs = np.mean([Wp[g * 4 + r] @ x for r in range(4)], axis=0)
        assert np.max(np.abs(lhs - rhs)) < 1e-13


ALL_CHECKS = [check_decode_vs_sdpa, check_decode_repeat_kv, check_decode_mqa_einsum, check_decode_mha_per_head,
              check_head_mapping_contiguous, check_identical_keys_mean_of_v, check_len1_and_len0,
              check_scale_limits, check_shift_and_permutation, check_prefill_vs_sdpa, check_prefill_rows,
              check_meanpool]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


# ---------------------------------------------------------------------------
# numbers printed on the pages

def _golden_sizes():
    rows = []
    with open(os.path.join(GOLDEN, "kv_cache_sizes.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            nums, cite = line.split("|", 1)
            L, K, d, b, tokens, expect = nums.split()
            rows.append((int(L), int(K), int(d), int(b), int(tokens), expect, cite.strip()))
    return rows


@pytest.mark.parametrize("row", _golden_sizes(), ids=lambda r: r[6][:40])
def test_kv_cache_size_matches_pages(row):
    L, K, d, b, tokens, expect, _ = row
    got = oracle.kv_cache_bytes_per_token(L, K, d, b) * tokens
    if expect.startswith("~"):
        e = float(expect[1:])
        digits = len(expect[1:].split("e")[0].replace(".", "").lstrip("0"))
        assert float(f"{got:.{digits - 1}e}") == pytest.approx(float(f"{e:.{digits - 1}e}"), rel=1e-12)
    else:
        assert got == int(expect)


def test_kv_cache_ratio_and_capacity_ledger():
    # GQA-8 (64 -> 8 heads) keeps 1/8 of the cache ("GQA 完全拆解", title and KV ledger)
    assert oracle.kv_cache_bytes_per_token(80, 64, 128, 2) == 8 * oracle.kv_cache_bytes_per_token(80, 8, 128, 2)
    # "分組查詢注意力", 關鍵引數: 2 x 64 x 2048 x 128 x 80 ~ 2.68e9 (an element count) and 1/8 with 8 KV heads
    mha = oracle.kv_cache_elements_per_layer_token(64, 128) * 2048 * 80
    assert round(mha / 1e9, 2) == 2.68
    assert mha // (oracle.kv_cache_elements_per_layer_token(8, 128) * 2048 * 80) == 8
    # capacity ledger: 64 GB free holds ~30 MHA requests at 4K and ~120 with 8 KV heads
    per_req_mha = oracle.kv_cache_bytes_per_token(32, 32, 128, 2) * 4096
    per_req_gqa = oracle.kv_cache_bytes_per_token(32, 8, 128, 2) * 4096
    assert round(64e9 / per_req_mha, -1) == 30
    assert round(64e9 / per_req_gqa, -1) == 120


# ---------------------------------------------------------------------------
# rounding to the storage type

BF16_CASES = [
    (1.0, 0x3F80), (1.0 + 2**-8, 0x3F80), (1.0 + 3 * 2**-8, 0x3F82), (1.0 + 2**-7, 0x3F81),
    (-2.5, 0xC020), (0.0, 0x0000), (-0.0, 0x8000), (3.3895313892515355e38, 0x7F7F),
    (2.0**128, 0x7F80), (-(2.0**129), 0xFF80), (2.0**-133, 0x0001), (2.0**-134, 0x0000),
    (1.5 * 2.0**-134, 0x0001), (2.0**-126, 0x0080), (float("nan"), 0x7FC0), (float("inf"), 0x7F80),
]


def test_bf16_rounding_known_patterns():
    x = np.array([c[0] for c in BF16_CASES])
    got = oracle.round_to(x, np.uint16)
    assert [int(v) for v in got] == [c[1] for c in BF16_CASES]


def test_bf16_rounding_matches_torch_on_float32_values():
    x = np.concatenate([rnd((20000,), 131, 1), rnd((20000,), 131, 2) * 1e-38, rnd((2000,), 131, 3) * 1e30])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_to(x32.astype(np.float64), np.uint16)
    assert np.array_equal(got, want)


def test_kv_append_writes_only_the_new_rows():
    B, K, S, d = 3, 2, 5, 4
    kc, vc = rnd((B, K, S, d), 141, 1), rnd((B, K, S, d), 141, 2)
    kn, vn = rnd((B, K, d), 141, 3), rnd((B, K, d), 141, 4)
    pos = np.array([0, 4, 7])  # the last one is out of range and ignored
    k2, v2 = oracle.kv_append(kc, vc, kn, vn, pos)
    assert np.array_equal(k2[0, :, 0], kn[0]) and np.array_equal(v2[1, :, 4], vn[1])
    mask = np.ones((B, K, S), bool)
    mask[0, :, 0] = mask[1, :, 4] = False
    assert np.array_equal(k2[mask], kc[mask]) and np.array_equal(v2[mask], vc[mask])
    assert np.array_equal(k2[2], kc[2])


# ---------------------------------------------------------------------------
# planted mistakes: every mutant of the oracle must fail at least one pin

MUTANTS = {
    "round_robin_heads": ("int g = h / G; /* contiguous grouping", "int g = h % jb->K; /* contiguous grouping"),
    "dropped_scale": ("s[t] = scale * acc;", "s[t] = acc;"),
    "unnormalised": ("out[i] /= Z;", "out[i] /= 1.0;"),
    "k_for_v": ("out[i] += w * widen_kv(v, kv_off", "out[i] += w * widen_kv(k, kv_off"),
    "no_max_subtraction": ("s[t] = exp(s[t] - m);", "s[t] = exp(s[t]);"),
    "ignores_seqlens": ("int64_t n = jb->seqlens[b];", "int64_t n = jb->S_max;"),
    "causal_excludes_diagonal": ("(int64_t)i + 1, jb->d,", "(int64_t)i, jb->d,"),
    "meanpool_divides_by_H": ("acc / (double)G;", "acc / (double)H;"),
    "meanpool_strided_groups": ("(int64_t)g * G + r) * inner", "(int64_t)g + (int64_t)r * K) * inner"),
    "transposed_prefill_q": ("(((int64_t)b * jb->S + i) * jb->H + h) * jb->d;\n  int64_t kv_off",
                             "(((int64_t)b * jb->S + (jb->S - 1 - i)) * jb->H + h) * jb->d;\n  int64_t kv_off"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
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
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"
