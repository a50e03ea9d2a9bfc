"""GPU parity of gqa_prefill_causal (tcgen05) with the float64 oracle."""
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


def make(B, S, H, K, d, seed):
    return {
        "q": synth.normal((B, S, H, d), synth.BF16, seed, 1),
        "k": synth.normal((B, S, K, d), synth.BF16, seed, 2),
        "v": synth.normal((B, S, K, d), synth.BF16, seed, 3),
    }


def run(gqa, inp, scale, S_max=None):
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    B, S, H, d = inp["q"].shape
    K = inp["k"].shape[2]
    out = Guarded((B, S, H, d), torch.bfloat16)
    kc = vc = None
    if S_max is not None:
        kc = dev(synth.cache(B * K, S_max, d, synth.BF16, 99, 7, np.zeros(B, np.int32), K).reshape(B, K, S_max, d))
        vc = dev(synth.cache(B * K, S_max, d, synth.BF16, 99, 8, np.zeros(B, np.int32), K).reshape(B, K, S_max, d))
    gqa.gqa_prefill_causal(out.t, q, k, v, scale, kc, vc)
    status = gqa.gqa_get_last_error()
    assert status == (0, 0), status
    assert out.intact(), "write outside the output buffer"
    return host(out.t), (host(kc) if kc is not None else None), (host(vc) if vc is not None else None)


SMALL = [
    # B, S, H, K, d
    (1, 128, 4, 1, 128),    # one query tile, MQA
    (2, 300, 8, 2, 128),    # ragged: neither 64 nor 128 divides S
    (1, 1000, 4, 4, 64),    # MHA, d = 64
    (2, 517, 12, 4, 128),   # G = 3
    (1, 64, 2, 2, 64),      # a single key tile
    (1, 1, 4, 2, 128),      # one token
    (4, 1024, 32, 8, 128),  # 512 head-pair units: several per persistent CTA
    (2, 1500, 16, 2, 64),   # G = 8 (four head pairs), d = 64, ragged, several units per CTA
    (1, 700, 16, 4, 128),   # ragged: a last key tile of 60 rows
    (2, 400, 12, 2, 128),   # G = 6: three head pairs per group
    (1, 260, 64, 1, 128),   # MQA, G = 64: 32 head pairs share every K/V tile
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}S{}H{}K{}d{}".format(*s))
def test_prefill_small_full_compare(gqa, shape):
    B, S, H, K, d = shape
    inp = make(B, S, H, K, d, 0x9F00 + S + H)
    scale = 1.0 / np.sqrt(d)
    got, _, _ = run(gqa, inp, scale)
    ref = oracle.prefill_causal(inp["q"], inp["k"], inp["v"], scale)
    assert_close(got, ref, str(shape))
    # row 0 sees only key 0: its output is v_0 exactly
    for h in range(H):
        assert np.array_equal(got[:, 0, h], inp["v"][:, 0, h // (H // K)])


@pytest.mark.parametrize("shape", [(2, 200, 8, 2, 128, 333), (1, 300, 4, 2, 64, 300), (2, 1024, 16, 4, 128, 1100),
                                   (2, 300, 12, 4, 128, 320)],
                         ids=["G4_tail72", "G2_d64_full", "G4_many_units", "G3_separate_write"])
def test_prefill_writes_the_cache(gqa, shape):
    # even G: the prefill kernel stores each key tile from shared memory (TMA
    # for whole 16-row groups, plain stores for the rest); odd G: a separate pass
    B, S, H, K, d, S_max = shape
    inp = make(B, S, H, K, d, 0x9F77 + S)
    got, kc, vc = run(gqa, inp, 0.1, S_max=S_max)
    want_k, want_v = oracle.prefill_cache_write(inp["k"], inp["v"], S_max,
                                                np.full((B, K, S_max, d), 0x7FC0, np.uint16),
                                                np.full((B, K, S_max, d), 0x7FC0, np.uint16))
    assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v)
    assert_close(got, oracle.prefill_causal(inp["q"], inp["k"], inp["v"], 0.1), str(shape))


def test_prefill_large_scores_stay_finite(gqa):
    # scores of several hundred (scale 1): the running max moves by more than
    # the rescale threshold many times within a row
    inp = make(1, 384, 4, 2, 128, 0x9F88)
    got, _, _ = run(gqa, inp, 1.0)
    ref = oracle.prefill_causal(inp["q"], inp["k"], inp["v"], 1.0)
    assert_close(got, ref, "scale 1")


def test_prefill_full_size_sampled(gqa):
    w = synth.PREFILL_WORKLOADS["causal_prefill_b4_s4096_h32_k8_d128"]
    inp = synth.prefill_inputs(w)
    scale = 1.0 / np.sqrt(w.d)
    got, kc, vc = run(gqa, inp, scale, S_max=w.S)
    assert np.all(np.isfinite(oracle.widen(got)))
    rng = np.random.default_rng(11)
    rows = np.concatenate([rng.integers(0, w.S, 40), [0, 1, 63, 64, 127, 128, 2047, w.S - 1]])
    sel = np.stack([rng.integers(0, w.B, rows.size), rows, rng.integers(0, w.H, rows.size)], 1).astype(np.int32)
    ref = oracle.prefill_causal(inp["q"], inp["k"], inp["v"], scale, sel=sel)
    assert_close(got[sel[:, 0], sel[:, 1], sel[:, 2]], ref, "causal prefill 4x4096x32x128")
    assert np.array_equal(kc, np.transpose(inp["k"], (0, 2, 1, 3)))
    assert np.array_equal(vc, np.transpose(inp["v"], (0, 2, 1, 3)))
