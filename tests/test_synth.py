"""The seeded input generator: deterministic, sliceable, N(0, 1), NaN past each length."""
import numpy as np

import synth


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: the published first outputs of the generator
    assert synth.draw(0, 0) == 0xE220A8397B1DCDAF
    assert synth.draw(0, 1) == 0x6E789E6AA1B965F4
    assert synth.draw(0, 2) == 0x06C45D188009454F


def test_normals_are_standard_and_sliceable():
    x = synth.normal((1 << 18,), synth.F64, 7, 1)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    key = synth.stream_key(7, 1)
    part = np.empty(1001, np.float64)
    synth._get().synth_normal(part.ctypes.data, synth.F64, key, 777, part.size, 3)
    assert np.array_equal(part, x[777:1778])


def test_dtypes_round_the_same_draws():
    x64 = synth.normal((4096,), synth.F64, 3, 2)
    x32 = synth.normal((4096,), synth.F32, 3, 2)
    xb = synth.normal((4096,), synth.BF16, 3, 2)
    assert np.array_equal(x32, x64.astype(np.float32))
    widened = (xb.astype(np.uint32) << 16).view(np.float32)
    assert np.max(np.abs(widened - x32) / np.maximum(np.abs(x32), 1e-30)) <= 2.0**-8


def test_cache_rows_past_length_are_nan():
    lens = np.array([3, 0, 5], np.int32)
    c = synth.cache(6, 5, 4, synth.F32, 9, 2, lens, 2)
    full = synth.normal((6, 5, 4), synth.F32, 9, 2)
    for u in range(6):
        n = lens[u // 2]
        assert np.array_equal(c[u, :n], full[u, :n])
        assert np.isnan(c[u, n:]).all()


def test_uniform_int_range_and_workload_lengths():
    v = synth.uniform_int(10000, 1024, 16384, 5, 4)
    assert v.min() >= 1024 and v.max() <= 16384
    w = synth.DECODE_WORKLOADS["ragged_70b_decode_b32_h64_k8_d128_s1k_16k"]
    lens = synth.seqlens_for(w)
    assert lens.shape == (32,) and lens.min() >= 1024 and lens.max() <= 16384


def test_permutation_is_a_seeded_permutation():
    p1 = synth.permutation(257, synth.SEED_BASE + 9, synth.STREAM_BLOCKS)
    p2 = synth.permutation(257, synth.SEED_BASE + 9, synth.STREAM_BLOCKS)
    p3 = synth.permutation(257, synth.SEED_BASE + 10, synth.STREAM_BLOCKS)
    assert np.array_equal(np.sort(p1), np.arange(257))
    assert np.array_equal(p1, p2) and not np.array_equal(p1, p3)


def test_page_scatters_every_valid_row_once():
    B, K, S, d, bs = 3, 2, 64, 8, 16
    lens = np.array([64, 5, 33], dtype=np.int32)
    kc = synth.cache(B * K, S, d, synth.BF16, 123, synth.STREAM_K, lens, K).reshape(B, K, S, d)
    vc = synth.cache(B * K, S, d, synth.BF16, 123, synth.STREAM_V, lens, K).reshape(B, K, S, d)
    pg = synth.page(kc, vc, lens, bs, spare_blocks=4, seed=123)
    table, kp = pg["block_table"], pg["k_pool"]
    need = (lens + bs - 1) // bs
    assert kp.shape == (int(need.sum()) + 4, K, bs, d) and table.shape == (B, S // bs)
    used = table[table >= 0]
    assert len(used) == need.sum() and len(np.unique(used)) == len(used)
    for b in range(B):
        assert (table[b, need[b]:] == -1).all()
        for i in range(need[b]):
            assert np.array_equal(kp[table[b, i]], kc[b, :, i * bs:(i + 1) * bs])
            assert np.array_equal(pg["v_pool"][table[b, i]], vc[b, :, i * bs:(i + 1) * bs])
    spare = np.setdiff1d(np.arange(kp.shape[0]), used)
    assert len(spare) == 4 and (kp[spare] == 0x7FC0).all()


def test_paged_inputs_map_the_append_row():
    # the block of each appended row (pos = len - 1) is mapped
    w = synth.DECODE_WORKLOADS["llama3_8b_decode_b8_h32_k8_d128_s8192"]
    pos = synth.seqlens_for(w) - 1
    kc = np.zeros((w.B, 1, w.S_max, 2), dtype=np.uint16)  # a tiny stand-in cache with the same lengths
    pg = synth.page(kc, kc, pos, 16, 2, w.seed, append_row=True)
    assert (pg["block_table"][np.arange(w.B), pos // 16] >= 0).all()


def test_int8_cache_codes_scales_and_padding():
    lens = np.array([5, 0], np.int32)
    c, s = synth.int8_cache(4, 8, 16, 77, synth.STREAM_K8, synth.STREAM_KSCALE, lens, 2, lo=0.01, hi=0.02)
    assert c.dtype == np.int8 and s.dtype == np.float32 and c.shape == (4, 8, 16) and s.shape == (4, 8)
    valid = np.zeros((4, 8), bool)
    valid[:2, :5] = True
    assert (c[valid] >= -127).all() and (c[valid] <= 127).all() and len(np.unique(c[valid])) > 50
    assert (s[valid] >= 0.01).all() and (s[valid] < 0.02).all()
    assert (c[~valid] == -128).all() and np.isnan(s[~valid]).all()
    c2, s2 = synth.int8_cache(4, 8, 16, 77, synth.STREAM_K8, synth.STREAM_KSCALE, lens, 2, lo=0.01, hi=0.02)
    assert np.array_equal(c, c2) and np.array_equal(s[valid], s2[valid])


def test_projection_inputs():
    w = synth.PROJ_WORKLOADS["kv_proj_decode_b8_t1_k8_d128_dm4096"]
    inp = synth.proj_inputs(w)
    assert inp["x"].shape == (8, 1, 4096) and inp["w_kv"].shape == (8, 256, 4096) and inp["w_kv"].dtype == np.uint16
    wf = (inp["w_kv"].astype(np.uint32) << 16).view(np.float32)
    assert abs(float(np.std(wf)) - 1 / 64) < 1e-3 and (inp["pos"] == 8191).all()
