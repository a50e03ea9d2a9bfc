"""GPU parity of gqa_kv_append and gqa_meanpool_kv with the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import Guarded, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    from kv_cache_02_b200 import gqa as g

    return g


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
@pytest.mark.parametrize("B,K,S_max,d", [(3, 2, 37, 128), (8, 8, 8192, 128), (1, 1, 5, 64), (5, 3, 100, 64)])
def test_append_bit_exact(gqa, dtype, B, K, S_max, d):
    seed = 0xA11 + B * 100 + K
    lens = synth.uniform_int(B, 0, S_max - 1, seed, 9)
    kc = synth.cache(B * K, S_max, d, dtype, seed, 2, lens, K).reshape(B, K, S_max, d)
    vc = synth.cache(B * K, S_max, d, dtype, seed, 3, lens, K).reshape(B, K, S_max, d)
    kn = synth.normal((B, K, d), dtype, seed, 5)
    vn = synth.normal((B, K, d), dtype, seed, 6)
    pos = lens.astype(np.int32)
    want_k, want_v = oracle.kv_append(kc, vc, kn, vn, pos)
    tk, tv = dev(kc), dev(vc)
    gqa.gqa_kv_append(tk, tv, dev(kn), dev(vn), dev(pos))
    assert gqa.gqa_get_last_error() == (0, 0)
    assert np.array_equal(host(tk).view(np.uint8), want_k.view(np.uint8))
    assert np.array_equal(host(tv).view(np.uint8), want_v.view(np.uint8))


def test_append_out_of_range_position_is_reported_not_written(gqa):
    B, K, S_max, d = 3, 2, 16, 128
    kc = synth.normal((B, K, S_max, d), synth.BF16, 77, 2)
    vc = synth.normal((B, K, S_max, d), synth.BF16, 77, 3)
    kn, vn = synth.normal((B, K, d), synth.BF16, 77, 5), synth.normal((B, K, d), synth.BF16, 77, 6)
    pos = np.array([3, S_max, -1], np.int32)
    tk, tv = dev(kc), dev(vc)
    gqa.gqa_kv_append(tk, tv, dev(kn), dev(vn), dev(pos))
    status, bits = gqa.gqa_get_last_error()
    assert status == gqa.GQA_ERR_DEVICE and bits & gqa.GQA_DEVERR_APPEND_POS
    want_k, want_v = oracle.kv_append(kc, vc, kn, vn, pos)
    assert np.array_equal(host(tk), want_k) and np.array_equal(host(tv), want_v)
    assert gqa.gqa_get_last_error() == (0, 0)  # cleared by the read


MEANPOOL_CASES = [
    # outer, H, K, inner
    (1, 64, 8, 128 * 8192),      # projection weights [H, d_k, d_model] of a 64-head model -> 8 KV heads
    (4, 32, 8, 512 * 128),       # per-head K tensor [B, H, S, d]
    (2, 12, 4, 1000),            # G = 3 (not a power of two)
    (3, 8, 8, 64),               # G = 1: a copy
    (2, 64, 1, 136),             # G = 64: MQA
    (3, 6, 2, 13),               # inner not a multiple of the vector width: scalar path
]


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
@pytest.mark.parametrize("outer,H,K,inner", MEANPOOL_CASES)
def test_meanpool_bit_exact(gqa, dtype, outer, H, K, inner):
    if outer * H * inner > 70_000_000 and dtype == synth.F32:
        pytest.skip("large f32 case covered by bf16")
    seed = 0xB00 + H * 7 + K
    src = synth.normal((outer, H, inner), dtype, seed, 1)
    want = oracle.round_to(oracle.meanpool_kv(src, K), src.dtype)
    dst = Guarded((outer, K, inner), torch.bfloat16 if dtype == synth.BF16 else torch.float32)
    gqa.gqa_meanpool_kv(dst.t, dev(src))
    torch.cuda.synchronize()
    assert dst.intact()
    assert np.array_equal(host(dst.t).view(np.uint8), want.view(np.uint8))


def test_meanpool_integer_heads_exact(gqa):
    # small integers x 2^-3 are exact in bf16: the mean is exact and the group
    # range is the one the GQA page prints ((g-1)h/G+1 .. gh/G, 1-based)
    outer, H, K, inner = 2, 16, 4, 256
    vals = (np.random.default_rng(3).integers(-64, 64, size=(outer, H, inner)) / 8.0).astype(np.float32)
    src = torch.from_numpy(vals).to(torch.bfloat16).cuda()
    dst = torch.empty((outer, K, inner), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_meanpool_kv(dst, src)
    want = torch.from_numpy(vals.astype(np.float64)).view(outer, K, H // K, inner).mean(2)
    assert torch.equal(dst.double().cpu(), want.to(torch.bfloat16).double())
