"""Decode calls back to back on one stream, each reading what the kernel
right before it wrote.

The decode kernels are launched as programmatic dependents of the kernel
before them: they set up and warm L2 with their first key rows while that
kernel finishes, and read their inputs only after the grid dependency. These
tests issue chains with no synchronisation between the calls and check every
output against the oracle:
  * a fused append followed at once by a decode that must see the appended
    row (the row held NaN before, so a stale read would poison the output),
    with the split combine between them and without it;
  * q and the lengths rewritten by a torch kernel right before a decode;
  * a prompt's K/V projected into the cache and decoded at once;
  * narrow-group and wide-group (tensor-core) calls alternating on one
    shared workspace, so each call's partials and work counter reuse the
    memory the previous call's combine is still reading.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    from kv_cache_02_b200 import gqa as g

    return g


def _cache(B, K, S_max, d, lens, seed):
    kc = synth.cache(B * K, S_max, d, synth.BF16, seed, 2, lens, K).reshape(B, K, S_max, d)
    vc = synth.cache(B * K, S_max, d, synth.BF16, seed, 3, lens, K).reshape(B, K, S_max, d)
    return kc, vc


@pytest.mark.parametrize("first_splits", [1, 3])
def test_append_then_decode_sees_the_new_row(gqa, first_splits):
    B, H, K, d, S_max = 4, 32, 8, 128, 1536
    pos = np.array([1535, 700, 0, 1023], np.int32)  # rows at pos hold NaN until the append
    seed = 0xC4A1 + first_splits
    kc, vc = _cache(B, K, S_max, d, pos, seed)
    q1 = synth.normal((B, H, d), synth.BF16, seed, 1)
    q2 = synth.normal((B, H, d), synth.BF16, seed, 7)
    kn, vn = synth.normal((B, K, d), synth.BF16, seed, 5), synth.normal((B, K, d), synth.BF16, seed, 6)
    tk, tv = dev(kc), dev(vc)
    tpos, tlen = dev(pos), dev(pos + 1)
    ws = torch.empty(max(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, n) for n in (0, first_splits, 3)),
                     dtype=torch.uint8, device="cuda")
    out1, out2 = (torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2))
    scale = 1.0 / np.sqrt(d)
    torch.cuda.synchronize()
    gqa.gqa_decode_append(out1, dev(q1), tk, tv, dev(kn), dev(vn), tpos, scale, first_splits, ws)
    gqa.gqa_decode(out2, dev(q2), tk, tv, tlen, scale, 3, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    kc2, vc2 = oracle.kv_append(kc, vc, kn, vn, pos)
    assert_close(host(out1), oracle.decode(q1, kc2, vc2, pos + 1, scale), "fused append + decode")
    assert_close(host(out2), oracle.decode(q2, kc2, vc2, pos + 1, scale), "decode right after the append")


def test_separate_append_then_decode(gqa):
    B, H, K, d, S_max = 2, 64, 1, 128, 4096  # G = 64: the separate append, then the wide-group kernel
    pos = np.array([4095, 2000], np.int32)
    seed = 0xC4B2
    kc, vc = _cache(B, K, S_max, d, pos, seed)
    q = synth.normal((B, H, d), synth.BF16, seed, 1)
    kn, vn = synth.normal((B, K, d), synth.BF16, seed, 5), synth.normal((B, K, d), synth.BF16, seed, 6)
    tk, tv = dev(kc), dev(vc)
    ws = torch.empty(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    tq, tkn, tvn, tpos, tlen = dev(q), dev(kn), dev(vn), dev(pos), dev(pos + 1)
    torch.cuda.synchronize()
    gqa.gqa_kv_append(tk, tv, tkn, tvn, tpos)
    gqa.gqa_decode(out, tq, tk, tv, tlen, 1.0 / np.sqrt(d), 0, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    kc2, vc2 = oracle.kv_append(kc, vc, kn, vn, pos)
    assert_close(host(out), oracle.decode(q, kc2, vc2, pos + 1, 1.0 / np.sqrt(d)), "append kernel, then decode")


def test_inputs_rewritten_by_torch_right_before(gqa):
    B, H, K, d, S_max = 4, 32, 8, 128, 2048
    lens = np.array([2048, 1500, 900, 64], np.int32)
    seed = 0xC4C3
    kc, vc = _cache(B, K, S_max, d, lens, seed)
    q = synth.normal((B, H, d), synth.BF16, seed, 1)
    tk, tv, tq, tl = dev(kc), dev(vc), dev(q), dev(lens)
    ws = torch.empty(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, 0), dtype=torch.uint8, device="cuda")
    out1, out2 = (torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2))
    cut = torch.tensor([100, 700, 0, 63], dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    torch.cuda.synchronize()
    gqa.gqa_decode(out1, tq, tk, tv, tl, scale, 0, ws)
    tq.mul_(-0.5)  # exact in bf16
    tl.sub_(cut)
    gqa.gqa_decode(out2, tq, tk, tv, tl, scale, 0, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    assert_close(host(out1), oracle.decode(q, kc, vc, lens, scale), "before the rewrite")
    q2 = oracle.round_to(oracle.widen(q) * -0.5, np.uint16)
    lens2 = lens - np.array([100, 700, 0, 63], np.int32)
    assert_close(host(out2), oracle.decode(q2, kc, vc, lens2, scale), "q and lengths rewritten just before")


def test_projection_then_decode(gqa):
    B, T, H, K, d, d_model, S_max = 2, 1024, 32, 8, 128, 256, 1024
    seed = 0xC4D4
    x = synth.normal((B, T, d_model), synth.BF16, seed, 8)
    # weights ~ N(0, 1/256) (a power-of-two scaling, exact in bf16): projected K/V of unit variance
    w = oracle.round_to(oracle.widen(synth.normal((K, 2 * d, d_model), synth.BF16, seed, 9)) / 16.0, np.uint16)
    nan_rows = np.zeros(B, np.int32)  # every row NaN until the projection writes it
    kc0, vc0 = _cache(B, K, S_max, d, nan_rows, seed)
    q = synth.normal((B, H, d), synth.BF16, seed, 1)
    tk, tv = dev(kc0), dev(vc0)
    assert gqa.gqa_kv_project_workspace_bytes(B, T, K, d, d_model) == 0  # one GEMM launch, no finalize pass
    ws = torch.empty(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    tx, tw, tq = dev(x), dev(w), dev(q)
    lens = np.full(B, T, np.int32)
    tl = dev(lens)
    torch.cuda.synchronize()
    gqa.gqa_kv_project_append(tk, tv, tx, tw)
    gqa.gqa_decode(out, tq, tk, tv, tl, 1.0 / np.sqrt(d), 0, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    kc, vc = oracle.kv_project_append(kc0, vc0, x, w, None)
    assert_close(host(out), oracle.decode(q, kc, vc, lens, 1.0 / np.sqrt(d)), "projection, then decode")


def test_narrow_and_wide_calls_share_a_workspace(gqa):
    cases = [
        # B, H, K, d, S_max, lens, num_splits
        (4, 32, 8, 128, 3000, (3000, 1, 2222, 1400), 0),
        (1, 64, 1, 128, 20000, (20000,), 0),      # wide group (MQA), one item per SM
        (2, 16, 2, 64, 5000, (5000, 4097), 9),
        (2, 128, 2, 128, 4100, (4100, 130), 0),   # wide group, two KV heads
    ]
    inputs, ws_need = [], 0
    for i, (B, H, K, d, S_max, lens, ns) in enumerate(cases):
        lens = np.array(lens, np.int32)
        kc, vc = _cache(B, K, S_max, d, lens, 0xC4E0 + i)
        q = synth.normal((B, H, d), synth.BF16, 0xC4E0 + i, 1)
        inputs.append((q, kc, vc, lens, ns, dev(q), dev(kc), dev(vc), dev(lens)))
        ws_need = max(ws_need, gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, ns))
    ws = torch.empty(ws_need, dtype=torch.uint8, device="cuda")
    rounds = 3
    outs = [[torch.empty(inp[5].shape, dtype=torch.bfloat16, device="cuda") for inp in inputs] for _ in range(rounds)]
    torch.cuda.synchronize()
    for r in range(rounds):
        for i, (_q, _k, _v, _l, ns, tq, tk, tv, tl) in enumerate(inputs):
            d = tq.shape[2]
            gqa.gqa_decode(outs[r][i], tq, tk, tv, tl, 1.0 / np.sqrt(d), ns, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    for i, (q, kc, vc, lens, ns, *_rest) in enumerate(inputs):
        d = q.shape[2]
        ref = oracle.decode(q, kc, vc, lens, 1.0 / np.sqrt(d))
        first = host(outs[0][i])
        assert_close(first, ref, f"case {i}")
        for r in range(1, rounds):
            assert np.array_equal(host(outs[r][i]), first), f"case {i}, round {r}: not bit for bit"
