"""GPU parity of gqa_kv_project_append (tcgen05 GEMM into the cache) with the oracle.

The written cache rows are compared with the float64 projection rounded
once to bf16 (within the bf16 tolerance); every other cache row must be
untouched (bit-exact). Decode-sized batches exercise the split of d_model
and the finalize pass, prompt-sized ones the direct epilogue.
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


def bf16_weights(shape, seed, scale):
    wf = synth.normal(shape, synth.F32, seed, 2) * np.float32(scale)
    return torch.from_numpy(wf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def run(gqa, x, w, S_max, pos):
    B, T, dm = x.shape
    K, two_d, _ = w.shape
    d = two_d // 2
    kc0 = synth.normal((B, K, S_max, d), synth.BF16, 77, 7)
    vc0 = synth.normal((B, K, S_max, d), synth.BF16, 77, 8)
    kc, vc = dev(kc0), dev(vc0)
    wsb = gqa.gqa_kv_project_workspace_bytes(B, T, K, d, dm)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if wsb else None
    gqa.gqa_kv_project_append(kc, vc, dev(x), dev(w), None if pos is None else dev(pos), ws)
    return host(kc), host(vc), kc0, vc0, gqa.gqa_get_last_error()


CASES = [
    # B, T, K, d, d_model, S_max, pos
    (8, 1, 8, 128, 4096, 64, (63, 0, 5, 17, 30, 40, 50, 60)),  # a decode step: the weight-streaming GEMV
    (3, 1, 2, 64, 512, 16, (0, 15, 7)),                         # d = 64
    (4, 4, 8, 128, 8192, 64, (0, 60, 33, 7)),                   # 16 tokens (two token tiles), the ring reused
    (2, 3, 4, 64, 1088, 32, (3, 29)),                           # a last stage of 64 columns
    (1, 1, 1, 64, 8192, 8, (7,)),                               # 128 W_KV rows: 8 CTAs, ring reused
    (2, 300, 4, 128, 1024, 320, (0, 20)),                        # a prompt: 300 tokens (ragged tiles)
    (1, 129, 1, 128, 256, 129, None),                            # MQA, pos None (0)
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}T{}K{}d{}dm{}".format(*c[:5]))
def test_projection_small(gqa, case):
    B, T, K, d, dm, S_max, pos = case
    x = synth.normal((B, T, dm), synth.BF16, 0x9E + T + dm, 1)
    w = bf16_weights((K, 2 * d, dm), 0x9E + K + d, 1 / np.sqrt(dm))
    pos = None if pos is None else np.array(pos, np.int32)
    kc, vc, kc0, vc0, status = run(gqa, x, w, S_max, pos)
    assert status == (0, 0)
    kv = oracle.kv_project(x, w)  # float64 [B, T, K, 2d]
    written = np.zeros(kc.shape[:3], bool)
    for b in range(B):
        p0 = 0 if pos is None else int(pos[b])
        written[b, :, p0:p0 + T] = True
        assert_close(np.transpose(kc[b, :, p0:p0 + T], (1, 0, 2)), kv[b, :, :, :d], f"K b={b}")
        assert_close(np.transpose(vc[b, :, p0:p0 + T], (1, 0, 2)), kv[b, :, :, d:], f"V b={b}")
    assert np.array_equal(kc[~written], kc0[~written]) and np.array_equal(vc[~written], vc0[~written])


def test_projection_out_of_range_positions(gqa):
    B, T, K, d, dm, S_max = 3, 4, 2, 128, 256, 10
    x = synth.normal((B, T, dm), synth.BF16, 0x9F, 1)
    w = bf16_weights((K, 2 * d, dm), 0x9F, 1 / 16)
    pos = np.array([6, 7, -1], np.int32)  # 6 + 4 fits exactly; 7 + 4 and -1 do not
    kc, vc, kc0, vc0, status = run(gqa, x, w, S_max, pos)
    assert status[0] == gqa.GQA_ERR_DEVICE and status[1] == gqa.GQA_DEVERR_APPEND_POS
    assert np.array_equal(kc[1:], kc0[1:]) and np.array_equal(vc[1:], vc0[1:])
    kv = oracle.kv_project(x, w)
    assert_close(np.transpose(kc[0, :, 6:10], (1, 0, 2)), kv[0, :, :, :d], "fits exactly")


@pytest.mark.parametrize("name", list(synth.PROJ_WORKLOADS))
def test_projection_full_size_sampled(gqa, name):
    w = synth.PROJ_WORKLOADS[name]
    inp = synth.proj_inputs(w)
    kc = torch.zeros((w.B, w.K, w.S_max, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    wsb = gqa.gqa_kv_project_workspace_bytes(w.B, w.T, w.K, w.d, w.d_model)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if wsb else None
    gqa.gqa_kv_project_append(kc, vc, dev(inp["x"]), dev(inp["w_kv"]), dev(inp["pos"]), ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    rng = np.random.default_rng(14)
    toks = [(b, int(i)) for b in range(w.B) for i in np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, 2)]))]
    xs = np.stack([inp["x"][b, i] for b, i in toks])
    kv = oracle.kv_project(xs, inp["w_kv"])  # [n, K, 2d]
    kch, vch = host(kc), host(vc)
    got_k = np.stack([kch[b, :, inp["pos"][b] + i] for b, i in toks])
    got_v = np.stack([vch[b, :, inp["pos"][b] + i] for b, i in toks])
    assert_close(got_k, kv[:, :, :w.d], name + " K")
    assert_close(got_v, kv[:, :, w.d:], name + " V")
