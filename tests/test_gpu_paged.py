"""GPU parity of the paged KV-cache calls with the float64 oracle.

The pools are the same seeded caches as the contiguous tests, scattered over
randomly placed blocks (unreferenced blocks and rows past each length hold
NaN; table entries past each sequence are -1). Besides the oracle, every
paged decode is compared bit for bit with the contiguous decode of the same
values: the paged kernels only change where a tile's rows come from, so the
arithmetic, and the result, must be identical.
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


def make(B, H, K, d, S_max, lens, seed):
    lens = np.asarray(lens, np.int32)
    return {
        "q": synth.normal((B, H, d), synth.BF16, seed, 1),
        "k_cache": synth.cache(B * K, S_max, d, synth.BF16, seed, 2, lens, K).reshape(B, K, S_max, d),
        "v_cache": synth.cache(B * K, S_max, d, synth.BF16, seed, 3, lens, K).reshape(B, K, S_max, d),
        "seqlens": lens,
    }


def workspace(nbytes):
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda") if nbytes else None


def run_paged(gqa, q, pg, lens, scale, num_splits):
    B, H, d = q.shape
    nb, K, bs, _ = pg["k_pool"].shape
    mb = pg["block_table"].shape[1]
    ws = workspace(gqa.gqa_decode_paged_workspace_bytes(B, H, K, d, bs, mb, num_splits))
    out = Guarded((B, H, d), torch.bfloat16)
    gqa.gqa_decode_paged(out.t, dev(q), dev(pg["k_pool"]), dev(pg["v_pool"]), dev(pg["block_table"]),
                         dev(lens.astype(np.int32)), scale, num_splits, ws)
    status = gqa.gqa_get_last_error()
    assert out.intact(), "write outside the output buffer"
    return host(out.t), status


def run_contiguous(gqa, inp, scale, num_splits):
    B, H, d = inp["q"].shape
    K, S_max = inp["k_cache"].shape[1:3]
    ws = workspace(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, num_splits))
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_decode(out, dev(inp["q"]), dev(inp["k_cache"]), dev(inp["v_cache"]), dev(inp["seqlens"]), scale,
                   num_splits, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    return host(out)


SMALL = [
    # B, H, K, d, S_max, lens, block sizes
    (3, 16, 4, 128, 320, (300, 1, 77), (16, 32, 64)),      # G = 4, ragged, one-key sequence
    (4, 64, 8, 128, 1024, (0, 999, 1024, 513), (16, 256)),  # G = 8, an empty sequence
    (2, 8, 8, 64, 192, (192, 65), (16, 48)),                # MHA, d = 64, a block size that is not a power of 2
    (2, 64, 1, 128, 768, (700, 129), (16, 128)),            # MQA (G = 64): the tensor-core wide path
    (3, 128, 2, 128, 256, (256, 1, 129), (16, 64)),         # G = 64: the tensor-core wide path, 16- and 64-row boxes
    (2, 128, 1, 128, 512, (500, 300), (32, 128)),           # G = 128: two 64-head slices
]
CASES = [(s, bs) for s in SMALL for bs in s[6]]


@pytest.mark.parametrize("num_splits", [0, 1, 3])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0][0]}H{c[0][1]}K{c[0][2]}d{c[0][3]}S{c[0][4]}bs{c[1]}")
def test_paged_decode_small(gqa, case, num_splits):
    (B, H, K, d, S_max, lens, _), bs = case
    inp = make(B, H, K, d, S_max, lens, 0x9A6E + B * 31 + H + K + d)
    pg = synth.page(inp["k_cache"], inp["v_cache"], inp["seqlens"], bs, spare_blocks=5, seed=0x9A6E + bs)
    scale = 1.0 / np.sqrt(d)
    got, status = run_paged(gqa, inp["q"], pg, inp["seqlens"], scale, num_splits)
    assert status == (0, 0)
    ref = oracle.decode_paged(inp["q"], pg["k_pool"], pg["v_pool"], pg["block_table"], inp["seqlens"], scale)
    assert_close(got, ref, f"{case} splits={num_splits}")
    # with the same split count, the same arithmetic as the contiguous cache:
    # identical bits (left to itself the planner gives a paged cache longer
    # splits, so the automatic counts may differ)
    if num_splits > 0:
        assert np.array_equal(got, run_contiguous(gqa, inp, scale, num_splits))


@pytest.mark.parametrize("bs", [16, 64])
@pytest.mark.parametrize("shape", [(3, 32, 8, 128, 256, (255, 16, 100)), (2, 64, 1, 128, 384, (300, 5))],
                         ids=["G4", "G64"])
def test_paged_decode_append(gqa, shape, bs):
    """gqa_decode_append_paged = gqa_kv_append_paged, then gqa_decode_paged over pos + 1 keys."""
    B, H, K, d, S_max, pos = shape
    seed = 0xA9E0 + H + bs
    inp = make(B, H, K, d, S_max, pos, seed)
    pos = np.asarray(pos, np.int32)
    pg = synth.page(inp["k_cache"], inp["v_cache"], pos, bs, spare_blocks=3, seed=seed, append_row=True)
    kn, vn = synth.normal((B, K, d), synth.BF16, seed, 5), synth.normal((B, K, d), synth.BF16, seed, 6)
    kp, vp, table = dev(pg["k_pool"]), dev(pg["v_pool"]), dev(pg["block_table"])
    ws = workspace(gqa.gqa_decode_paged_workspace_bytes(B, H, K, d, bs, table.shape[1], 0))
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / np.sqrt(d)
    gqa.gqa_decode_append_paged(out, dev(inp["q"]), kp, vp, dev(kn), dev(vn), table, dev(pos), scale, 0, ws)
    assert gqa.gqa_get_last_error() == (0, 0)
    kp_ref, vp_ref = oracle.kv_append_paged(pg["k_pool"], pg["v_pool"], kn, vn, pg["block_table"], pos)
    assert np.array_equal(host(kp), kp_ref) and np.array_equal(host(vp), vp_ref)
    ref = oracle.decode_paged(inp["q"], kp_ref, vp_ref, pg["block_table"], pos + 1, scale)
    assert_close(host(out), ref, f"{shape} bs={bs}")


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32], ids=["bf16", "f32"])
def test_kv_append_paged_bit_exact(gqa, dtype):
    B, K, d, S_max, bs = 4, 2, 64, 128, 16
    lens = np.array([0, 17, 64, 127], np.int32)
    seed = 0xA99 + dtype
    kc = synth.cache(B * K, S_max, d, dtype, seed, 2, lens, K).reshape(B, K, S_max, d)
    vc = synth.cache(B * K, S_max, d, dtype, seed, 3, lens, K).reshape(B, K, S_max, d)
    pg = synth.page(kc, vc, lens, bs, spare_blocks=2, seed=seed, append_row=True)
    kn, vn = synth.normal((B, K, d), dtype, seed, 5), synth.normal((B, K, d), dtype, seed, 6)
    kp, vp = dev(pg["k_pool"]), dev(pg["v_pool"])
    gqa.gqa_kv_append_paged(kp, vp, dev(kn), dev(vn), dev(pg["block_table"]), dev(lens))
    assert gqa.gqa_get_last_error() == (0, 0)
    kp_ref, vp_ref = oracle.kv_append_paged(pg["k_pool"], pg["v_pool"], kn, vn, pg["block_table"], lens)
    assert np.array_equal(host(kp).view(np.uint8), kp_ref.view(np.uint8))
    assert np.array_equal(host(vp).view(np.uint8), vp_ref.view(np.uint8))


def test_paged_errors_are_reported(gqa):
    B, H, K, d, S_max, bs = 2, 16, 4, 128, 128, 16
    lens = np.array([100, 50], np.int32)
    inp = make(B, H, K, d, S_max, lens, 0xE44)
    pg = synth.page(inp["k_cache"], inp["v_cache"], lens, bs, spare_blocks=1, seed=0xE44)
    # a table entry inside the length that points outside the pool
    bad = pg["block_table"].copy()
    bad[1, 2] = pg["k_pool"].shape[0] + 7
    got, status = run_paged(gqa, inp["q"], dict(pg, block_table=bad), lens, 0.1, 0)
    assert status[0] == gqa.GQA_ERR_DEVICE and status[1] & gqa.GQA_DEVERR_BLOCK
    # entries past the length are never read: -1 there is fine
    assert (pg["block_table"][1, 4:] == -1).all()
    got, status = run_paged(gqa, inp["q"], pg, lens, 0.1, 0)
    assert status == (0, 0)
    # append: a position past the capacity, and a block outside the pool
    kp, vp = dev(pg["k_pool"]), dev(pg["v_pool"])
    kn = dev(synth.normal((B, K, d), synth.BF16, 1, 5))
    gqa.gqa_kv_append_paged(kp, vp, kn, kn, dev(pg["block_table"]), dev(np.array([S_max, 3], np.int32)))
    st = gqa.gqa_get_last_error()
    assert st[0] == gqa.GQA_ERR_DEVICE and st[1] & gqa.GQA_DEVERR_APPEND_POS
    gqa.gqa_kv_append_paged(kp, vp, kn, kn, dev(bad), dev(np.array([3, 40], np.int32)))
    st = gqa.gqa_get_last_error()
    assert st[0] == gqa.GQA_ERR_DEVICE and st[1] & gqa.GQA_DEVERR_BLOCK


# ---------------------------------------------------------------------------
# full size, in the configuration the benchmark times


@pytest.mark.parametrize("name", list(synth.PAGED_WORKLOADS))
def test_paged_full_size_sampled(gqa, name):
    pw = synth.PAGED_WORKLOADS[name]
    w = synth.DECODE_WORKLOADS[pw.base]
    inp = synth.paged_inputs(pw)
    scale = 1.0 / np.sqrt(w.d)
    B, H, K, d = w.B, w.H, w.K, w.d
    table = inp["block_table"]
    kp, vp = dev(inp["k_pool"]), dev(inp["v_pool"])
    ws = workspace(gqa.gqa_decode_paged_workspace_bytes(B, H, K, d, pw.block_size, table.shape[1], 0))
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    if w.append:
        pos = inp["pos"]
        gqa.gqa_decode_append_paged(out, dev(inp["q"]), kp, vp, dev(inp["k_new"]), dev(inp["v_new"]), dev(table),
                                    dev(pos), scale, 0, ws)
        k_pool, v_pool = oracle.kv_append_paged(inp["k_pool"], inp["v_pool"], inp["k_new"], inp["v_new"], table, pos)
        lens = pos + 1
    else:
        gqa.gqa_decode_paged(out, dev(inp["q"]), kp, vp, dev(table), dev(inp["seqlens"]), scale, 0, ws)
        k_pool, v_pool, lens = inp["k_pool"], inp["v_pool"], inp["seqlens"]
    assert gqa.gqa_get_last_error() == (0, 0)
    got = host(out)
    rng = np.random.default_rng(11)
    sel = np.stack([rng.integers(0, B, 24), rng.integers(0, H, 24)], axis=1)
    sel[0], sel[1] = (0, 0), (B - 1, H - 1)
    ref = oracle.decode_paged(inp["q"], k_pool, v_pool, table, lens, scale, sel=sel)
    assert_close(got[sel[:, 0], sel[:, 1]], ref, name)
    if w.append:  # the appended rows, bit for bit
        assert np.array_equal(host(kp)[table[np.arange(B), pos // pw.block_size], :, pos % pw.block_size],
                              inp["k_new"])


def test_paged_decode_graph_replay(gqa):
    """gqa_decode_append_paged captured in a CUDA graph and replayed gives the
    eager call's bits (the warp-wide paged producer and the work counter's
    reset at the end of every launch)."""
    pw = synth.PAGED_WORKLOADS["paged_llama3_8b_decode_b8_h32_k8_d128_s8192_bs16"]
    w = synth.DECODE_WORKLOADS[pw.base]
    inp = synth.paged_inputs(pw)
    B, H, K, d = w.B, w.H, w.K, w.d
    kp, vp, table = dev(inp["k_pool"]), dev(inp["v_pool"]), dev(inp["block_table"])
    q, kn, vn, pos = dev(inp["q"]), dev(inp["k_new"]), dev(inp["v_new"]), dev(inp["pos"])
    ws = workspace(gqa.gqa_decode_paged_workspace_bytes(B, H, K, d, pw.block_size, table.shape[1], 0))
    out, ref = torch.empty_like(q), torch.empty_like(q)
    scale = 1.0 / np.sqrt(d)

    def call(o):
        gqa.gqa_decode_append_paged(o, q, kp, vp, kn, vn, table, pos, scale, 0, ws)

    call(out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(out)
    for rep in range(3):
        q.copy_(dev(synth.normal((B, H, d), synth.BF16, w.seed, 30 + rep)))
        out.fill_(float("nan"))
        g.replay()
        call(ref)
        assert gqa.gqa_get_last_error() == (0, 0)
        assert np.array_equal(host(out), host(ref)), f"replay {rep}"
    del g
