"""GPU parity of gqa_prefill_causal_varlen (tcgen05) with the float64 oracle.

Packed batches of prompts of different lengths (ragged against both the
128-row query tiles and the 64-key tiles, single-token and empty prompts)
are compared element by element with the oracle, which prefills every
sequence on its own; the cache rows are compared bit for bit. Output rows
are surrounded by sentinel bytes so that a write past a sequence shows.
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


def make(lens, H, K, d, seed):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    return {"cu": cu, "q": synth.normal((T, H, d), synth.BF16, seed, 1),
            "k": synth.normal((T, K, d), synth.BF16, seed, 2), "v": synth.normal((T, K, d), synth.BF16, seed, 3)}


def run(gqa, inp, scale, S_max=None):
    T, H, d = inp["q"].shape
    K = inp["k"].shape[1]
    B = len(inp["cu"]) - 1
    out = Guarded((T, H, d), torch.bfloat16)
    kc = vc = None
    if S_max is not None:
        kc = dev(synth.cache(B * K, S_max, d, synth.BF16, 98, 7, np.zeros(B, np.int32), K).reshape(B, K, S_max, d))
        vc = dev(synth.cache(B * K, S_max, d, synth.BF16, 98, 8, np.zeros(B, np.int32), K).reshape(B, K, S_max, d))
    gqa.gqa_prefill_causal_varlen(out.t, dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["cu"]), scale, kc, vc)
    status = gqa.gqa_get_last_error()
    assert out.intact(), "write outside the output buffer"
    return host(out.t), status, (host(kc) if kc is not None else None), (host(vc) if vc is not None else None)


CASES = [
    # lens, H, K, d
    ((300, 1, 129, 64, 517), 8, 2, 128),   # ragged, a single-token prompt
    ((128, 0, 256, 7), 4, 1, 128),         # an empty prompt, MQA
    ((1000, 33), 4, 4, 64),                # MHA, d = 64
    ((200, 200, 200), 12, 4, 128),         # equal lengths, G = 3
    (tuple(int(x) for x in np.random.default_rng(5).integers(0, 150, 40)), 4, 2, 64),  # 40 short prompts
    ((900, 1100, 37, 640, 1500), 32, 8, 128),  # 560 head-pair units: several per persistent CTA
    ((300, 0, 45, 129), 64, 1, 128),       # MQA (G = 64, 32 head pairs) with an empty prompt
    ((77, 400), 12, 2, 64),                # G = 6, d = 64
    (tuple(int(x) for x in np.random.default_rng(9).integers(0, 300, 256)), 8, 2, 64),  # 256 prompts: the
    # most that the per-CTA unit list takes, 1 to 3 query tiles each
    (tuple(int(x) for x in np.random.default_rng(11).integers(0, 60, 300)), 4, 2, 64),  # 300 prompts: the
    # sequence-major order
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "lens{}H{}K{}d{}".format(len(c[0]), *c[1:]))
def test_varlen_prefill(gqa, case):
    lens, H, K, d = case
    inp = make(lens, H, K, d, 0x7A + H + sum(lens))
    scale = 1.0 / np.sqrt(d)
    S_max = max(lens) + 16
    got, status, kc, vc = run(gqa, inp, scale, S_max)
    assert status == (0, 0)
    ref = oracle.prefill_causal_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], scale)
    assert_close(got, ref, str(case))
    B = len(lens)
    kc0 = synth.cache(B * K, S_max, d, synth.BF16, 98, 7, np.zeros(B, np.int32), K).reshape(B, K, S_max, d)
    vc0 = synth.cache(B * K, S_max, d, synth.BF16, 98, 8, np.zeros(B, np.int32), K).reshape(B, K, S_max, d)
    rk, rv = oracle.prefill_cache_write_varlen(inp["k"], inp["v"], inp["cu"], S_max, kc0, vc0)
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv)


def test_varlen_equals_fixed_length(gqa):
    """Equal lengths packed: identical bits to gqa_prefill_causal on the [B, S] layout."""
    B, S, H, K, d = 3, 300, 8, 2, 128
    inp = make([S] * B, H, K, d, 0x7B)
    got, status, _, _ = run(gqa, inp, 0.09)
    assert status == (0, 0)
    out = torch.empty((B, S, H, d), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_prefill_causal(out, dev(inp["q"].reshape(B, S, H, d)), dev(inp["k"].reshape(B, S, K, d)),
                           dev(inp["v"].reshape(B, S, K, d)), 0.09)
    assert gqa.gqa_get_last_error() == (0, 0)
    assert np.array_equal(got, host(out).reshape(B * S, H, d))


def test_varlen_bad_offsets_reported(gqa):
    inp = make((100, 50), 4, 2, 128, 0x7C)
    inp["cu"] = np.array([0, 120, 90], np.int32)  # decreasing: sequence 1 runs backwards
    got, status, _, _ = run(gqa, inp, 0.1)
    assert status[0] == gqa.GQA_ERR_DEVICE and status[1] & gqa.GQA_DEVERR_SEQLEN


@pytest.mark.parametrize("name", list(synth.VARLEN_WORKLOADS))
def test_varlen_full_size_sampled(gqa, name):
    w = synth.VARLEN_WORKLOADS[name]
    inp = synth.varlen_inputs(w)
    cu = inp["cu_seqlens"]
    T = int(cu[-1])
    scale = 1.0 / np.sqrt(w.d)
    out = torch.empty((T, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((w.B, w.K, w.S_max, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    gqa.gqa_prefill_causal_varlen(out, dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(cu), scale, kc, vc)
    assert gqa.gqa_get_last_error() == (0, 0)
    got = host(out)
    rng = np.random.default_rng(13)
    for b in range(w.B):  # sampled rows of every sequence, first and last included
        rows = np.unique(np.concatenate([[0, inp["lens"][b] - 1], rng.integers(0, inp["lens"][b], 3)]))
        sel = np.array([(0, int(r), int(h)) for r in rows for h in (0, w.H - 1)], np.int32)
        s = slice(cu[b], cu[b + 1])
        ref = oracle.prefill_causal(inp["q"][None, s], inp["k"][None, s], inp["v"][None, s], scale, sel=sel)
        assert_close(got[s][sel[:, 1], sel[:, 2]], ref, f"{name} sequence {b}")
    b = w.B - 1
    assert np.array_equal(host(kc)[b, :, :inp["lens"][b]], np.transpose(inp["k"][cu[b]:cu[b + 1]], (1, 0, 2)))
