"""The failure path of a bounded wait, on the GPU.

Every mbarrier wait in the pipelined kernels gives up after a time limit,
sets GQA_DEVERR_TIMEOUT in the device error word, lets the loads its CTA has
in flight land and returns: nothing traps, so the CUDA context stays usable.

This test loads a second build of the same sources, libgqa_waittest.so, in
which the limit is 20 ms and the first CTA of a narrow-group decode never
issues the load of its first work item's second tile. That stage's full
barrier is never completed by anything, so the consumers' wait for it runs
out (and then the producer's wait for the stage they never release, and its
final wait for the tile it never loaded). The call must report the timeout
through gqa_get_last_error, and afterwards a normal decode on the same stream
(the product library) must still match the oracle.
"""
import ctypes
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu

GQA_BF16 = 1


def _wait_test_lib():
    from kv_cache_02_b200 import build

    path = build.WAIT_TEST_LIB
    assert os.path.exists(path), f"{path} is missing: build it with `python -m kv_cache_02_b200.build`"
    lib = ctypes.CDLL(path)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.gqa_decode_workspace_bytes.restype = SZ
    lib.gqa_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.gqa_decode.restype = I
    lib.gqa_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P, SZ, I, P]
    lib.gqa_get_last_error.restype = I
    lib.gqa_get_last_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    return lib


def test_expired_wait_is_reported_and_the_context_stays_usable():
    from kv_cache_02_b200 import gqa

    B, H, K, d, S_max = 2, 16, 4, 128, 1024
    lens = np.array([1024, 700], np.int32)
    seed = 0x71E0
    kc = synth.cache(B * K, S_max, d, synth.BF16, seed, 2, lens, K).reshape(B, K, S_max, d)
    vc = synth.cache(B * K, S_max, d, synth.BF16, seed, 3, lens, K).reshape(B, K, S_max, d)
    q = synth.normal((B, H, d), synth.BF16, seed, 1)
    tq, tk, tv, tl = dev(q), dev(kc), dev(vc), dev(lens)
    scale = 1.0 / np.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream
    vp = ctypes.c_void_p

    wl = _wait_test_lib()
    ws_bytes = wl.gqa_decode_workspace_bytes(B, H, K, S_max, d, 1)  # one split: 16 tiles in the first item
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.zeros((B, H, d), dtype=torch.bfloat16, device="cuda")
    t0 = time.monotonic()
    rc = wl.gqa_decode(vp(out.data_ptr()), vp(tq.data_ptr()), vp(tk.data_ptr()), vp(tv.data_ptr()),
                       vp(tl.data_ptr()), B, H, K, S_max, d, ctypes.c_float(scale), 1, vp(ws.data_ptr()),
                       ws.numel(), GQA_BF16, vp(stream))
    assert rc == 0  # the launch itself is fine
    bits = ctypes.c_uint32(0)
    status = wl.gqa_get_last_error(vp(stream), ctypes.byref(bits))  # synchronizes the stream
    elapsed = time.monotonic() - t0
    assert status == gqa.GQA_ERR_DEVICE and bits.value & gqa.GQA_DEVERR_TIMEOUT, (status, bits.value)
    assert elapsed < 10.0  # three 20 ms limits, not a hang
    # the word is cleared by the read
    status2 = wl.gqa_get_last_error(vp(stream), ctypes.byref(bits))
    assert status2 == 0 and bits.value == 0

    # the context is intact: the product library's decode on the same stream matches the oracle
    torch.cuda.synchronize()
    ws2 = torch.empty(max(gqa.gqa_decode_workspace_bytes(B, H, K, S_max, d, 0), 16), dtype=torch.uint8,
                      device="cuda")
    out2 = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_decode(out2, tq, tk, tv, tl, scale, 0, ws2)
    assert gqa.gqa_get_last_error() == (0, 0)
    assert_close(host(out2), oracle.decode(q, kc, vc, lens, scale), "decode after an expired wait")
