"""gqa_decode_noalloc checked against gqa_decode and the oracle.

Some callers cannot allocate device memory when they decode: a plugin whose
host framework owns every device allocation, or a serving loop that forbids
allocation after start-up. gqa_decode_noalloc serves them by keeping the
split-KV partials in a static scratch array of the library instead of a
workspace the caller allocates. This test calls it through the C ABI twice in
a row, on two inputs that both need split-KV scratch, and compares each output
with gqa_decode's (caller workspace) within the decode tolerance and with the
float64 oracle. After one warm-up call (which may load the array), the two
calls must leave the device's free memory unchanged. It sits in a file of its
own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import TOL, assert_close, dev, host

pytestmark = pytest.mark.gpu

GQA_BF16 = 1


def _host_inputs(B, H, K, d, S_max, lens, seed):
    lens = np.asarray(lens, np.int32)
    kc = synth.cache(B * K, S_max, d, synth.BF16, seed, 2, lens, K).reshape(B, K, S_max, d)
    vc = synth.cache(B * K, S_max, d, synth.BF16, seed, 3, lens, K).reshape(B, K, S_max, d)
    return synth.normal((B, H, d), synth.BF16, seed, 1), kc, vc, lens


def _noalloc(lib, out, q, kc, vc, lens, scale, num_splits):
    B, H, d = q.shape
    K, S_max = kc.shape[1], kc.shape[2]
    vp = ctypes.c_void_p
    return lib.gqa_decode_noalloc(vp(out.data_ptr()), vp(q.data_ptr()), vp(kc.data_ptr()), vp(vc.data_ptr()),
                                  vp(lens.data_ptr()), B, H, K, S_max, d, ctypes.c_float(scale), num_splits,
                                  GQA_BF16, vp(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    from kv_cache_02_b200 import gqa

    lib = gqa.library()
    cases = [
        # B, H, K, d, S_max, lens, num_splits, seed
        (4, 32, 8, 128, 4096, (4096, 3000, 1, 2222), 0, 0x2A01),
        (2, 64, 8, 128, 8192, (8192, 5000), 6, 0x2A02),
    ]
    refs, outs, hosts = [], [], []
    for B, H, K, d, S_max, lens, ns, seed in cases:
        hq, hk, hv, hl = _host_inputs(B, H, K, d, S_max, lens, seed)
        q, kc, vc, ln = dev(hq), dev(hk), dev(hv), dev(hl)
        need = gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, ns)
        assert 0 < need <= gqa.GQA_NOALLOC_SCRATCH_BYTES  # the split-KV scratch is really used
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(q)
        gqa.gqa_decode(ref, q, kc, vc, ln, 1.0 / np.sqrt(d), ns, ws)
        refs.append(ref)
        outs.append((torch.full_like(q, float("nan")), q, kc, vc, ln, 1.0 / np.sqrt(d), ns))
        hosts.append((hq, hk, hv, hl, 1.0 / np.sqrt(d)))
    # a warm-up call: it may load the part of the library that holds the scratch
    warm = torch.empty_like(outs[0][1])
    assert _noalloc(lib, warm, *outs[0][1:]) == 0
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    # the two no-alloc calls back to back on one stream
    for out, q, kc, vc, ln, scale, ns in outs:
        assert _noalloc(lib, out, q, kc, vc, ln, scale, ns) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before, "the no-alloc calls changed the device's free memory"
    assert gqa.gqa_get_last_error() == (0, 0)
    tol_abs, tol_rel = TOL["bf16"]
    for ref, (out, *_rest), (hq, hk, hv, hl, scale) in zip(refs, outs, hosts):
        r = host(ref).astype(np.uint32) << 16
        o = host(out).astype(np.uint32) << 16
        r, o = r.view(np.float32).astype(np.float64), o.view(np.float32).astype(np.float64)
        assert np.all(np.isfinite(o))
        err = float(np.max(np.abs(o - r)))
        assert err <= tol_abs and err / float(np.max(np.abs(r))) <= tol_rel, err
        assert_close(host(out), oracle.decode(hq, hk, hv, hl, scale), "no-alloc decode vs the oracle")


def test_noalloc_rejects_requests_beyond_its_scratch():
    from kv_cache_02_b200 import gqa

    lib = gqa.library()
    B, H, K, d, S_max, ns = 32, 64, 8, 128, 16384, 64
    assert gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, ns) > gqa.GQA_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never touched: the size check comes first
    rc = lib.gqa_decode_noalloc(fake, fake, fake, fake, fake, B, H, K, S_max, d, ctypes.c_float(0.1), ns, GQA_BF16,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == gqa.GQA_ERR_SCRATCH_LIMIT
