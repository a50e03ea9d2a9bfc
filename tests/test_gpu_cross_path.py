"""Different kernels of the library on the same attention problem.

"GQA 完全拆解", section GQA：插值在 MHA 与 MQA 之间的分组共享: GQA with one group
per head is MHA and with one group for all heads is MQA, so the same
numbers can be reached along different paths. Two ties between kernels that
share no code:
  * causal prefill (tcgen05, one 128-row query tile per CTA) against decode
    (mma.sync, persistent ring): row i of a prefill is the decode of query i
    over the first i + 1 cached keys, the cache being the one the prefill
    wrote. Rows at tile edges are checked.
  * MQA (K = 1, G = 64: the tcgen05 wide-group decode) against the same
    problem written as K = 8 groups of 8 heads whose KV heads are all copies
    of the single one (the narrow-group mma.sync decode).
Each output is also compared with the float64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import TOL, assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    from kv_cache_02_b200 import gqa as g

    return g


def _close(a, b, what):
    """Two bf16 results of the same quantity agree within the decode tolerance."""
    fa, fb = oracle.widen(a), oracle.widen(b)
    tol_abs, tol_rel = TOL["bf16"]
    err = float(np.max(np.abs(fa - fb)))
    assert err <= tol_abs and err / float(np.max(np.abs(fb))) <= tol_rel, f"{what}: {err:.3e}"


@pytest.mark.parametrize("shape", [(2, 640, 16, 4, 128), (1, 300, 8, 8, 64)], ids=["G4d128", "G1d64"])
def test_prefill_rows_equal_decodes_over_the_prefix(gqa, shape):
    B, S, H, K, d = shape
    seed = 0xC205 + S
    q = synth.normal((B, S, H, d), synth.BF16, seed, 1)
    k = synth.normal((B, S, K, d), synth.BF16, seed, 2)
    v = synth.normal((B, S, K, d), synth.BF16, seed, 3)
    scale = 1.0 / np.sqrt(d)
    tq, tk, tv = dev(q), dev(k), dev(v)
    out = torch.empty_like(tq)
    kc = torch.full((B, K, S, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    gqa.gqa_prefill_causal(out, tq, tk, tv, scale, kc, vc)
    rows = sorted({0, 1, 63, 64, 127, 128, 129, 255, 256, S // 2, S - 2, S - 1})
    rows = [i for i in rows if i < S]
    pf = host(out)
    ws = torch.empty(max(gqa.gqa_decode_workspace_bytes(B, H, K, S, d, 0), 16), dtype=torch.uint8, device="cuda")
    for i in rows:
        qi = tq[:, i].contiguous()  # [B, H, d]: query row i of every sequence
        lens = torch.full((B,), i + 1, dtype=torch.int32, device="cuda")
        dec = torch.empty_like(qi)
        gqa.gqa_decode(dec, qi, kc, vc, lens, scale, 0, ws)
        got_dec = host(dec)
        _close(pf[:, i], got_dec, f"prefill row {i} vs decode over {i + 1} keys")
        ref = oracle.decode(q[:, i], np.transpose(k, (0, 2, 1, 3)), np.transpose(v, (0, 2, 1, 3)),
                            np.full(B, i + 1, np.int32), scale)
        assert_close(got_dec, ref, f"decode row {i}")
        assert_close(pf[:, i], ref, f"prefill row {i}")
    assert gqa.gqa_get_last_error() == (0, 0)


@pytest.mark.parametrize("S_max,lens", [(3000, (3000, 1777)), (131072 // 16, (8192, 1))])
def test_mqa_wide_path_equals_duplicated_heads_on_the_narrow_path(gqa, S_max, lens):
    B, H, d = len(lens), 64, 128
    lens = np.array(lens, np.int32)
    seed = 0xC20A + S_max
    kc1 = synth.cache(B, S_max, d, synth.BF16, seed, 2, lens, 1).reshape(B, 1, S_max, d)
    vc1 = synth.cache(B, S_max, d, synth.BF16, seed, 3, lens, 1).reshape(B, 1, S_max, d)
    q = synth.normal((B, H, d), synth.BF16, seed, 1)
    scale = 1.0 / np.sqrt(d)
    tq, tl = dev(q), dev(lens)
    outs = []
    for K in (1, 8):  # G = 64 (wide-group tcgen05 kernel), then G = 8 (narrow-group kernel)
        tk = dev(np.ascontiguousarray(np.repeat(kc1, K, axis=1)))
        tv = dev(np.ascontiguousarray(np.repeat(vc1, K, axis=1)))
        ws = torch.empty(max(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, 0), 16), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty_like(tq)
        gqa.gqa_decode(out, tq, tk, tv, tl, scale, 0, ws)
        outs.append(host(out))
        del tk, tv
    assert gqa.gqa_get_last_error() == (0, 0)
    _close(outs[0], outs[1], "K = 1 (wide) vs K = 8 copies (narrow)")
    ref = oracle.decode(q, kc1, vc1, lens, scale)
    assert_close(outs[0], ref, "MQA, wide path")
    assert_close(outs[1], ref, "MQA as duplicated groups, narrow path")
