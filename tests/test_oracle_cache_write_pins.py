"""Pins for the oracle's prompt cache write (the fixed-length prefill form).

The prompt's keys and values are written to the cache once, row t of KV head
g at key t ("GQA 完全拆解", section 解码推理的内存账本: the prompt's K/V go
into the cache and every later step reads them from there). The oracle's
`prefill_cache_write` turns k/v [B, S, K, d] into caches [B, K, S_max, d].
Checked here by an explicit loop over (b, t, g), by the rows it must leave
alone, against the varlen form when every sequence has the same length, and
by planted mistakes that each must fail a check. S = K in the loop check, so
that a transposed pair of axes still has the right shape and is caught by
value, not by a shape error.
"""
import numpy as np

import oracle
import synth


def rnd(shape, seed, stream):
    return synth.normal(shape, synth.F64, seed, stream)


def _loop_check(impl, B=2, S=3, K=3, d=4, S_max=5):
    """Row t of (b, g) is k[b, t, g] (and v's); rows >= S keep their sentinel."""
    k, v = rnd((B, S, K, d), 41, 2), rnd((B, S, K, d), 41, 3)
    kc0 = np.full((B, K, S_max, d), -5.0)
    vc0 = np.full((B, K, S_max, d), -9.0)
    kc, vc = impl(k, v, S_max, kc0, vc0)
    if kc.shape != (B, K, S_max, d) or vc.shape != (B, K, S_max, d):
        return False
    for b in range(B):
        for g in range(K):
            for t in range(S_max):
                if t < S:
                    if not (np.array_equal(kc[b, g, t], k[b, t, g]) and np.array_equal(vc[b, g, t], v[b, t, g])):
                        return False
                elif not ((kc[b, g, t] == -5.0).all() and (vc[b, g, t] == -9.0).all()):
                    return False
    # the inputs' own buffers are not modified
    return bool((kc0 == -5.0).all() and (vc0 == -9.0).all())


def test_rows_by_explicit_loop():
    assert _loop_check(oracle.prefill_cache_write)
    assert _loop_check(oracle.prefill_cache_write, B=1, S=4, K=2, d=8, S_max=4)  # a full cache


def test_default_caches_are_zero_past_the_prompt():
    k, v = rnd((2, 3, 2, 4), 42, 2), rnd((2, 3, 2, 4), 42, 3)
    kc, vc = oracle.prefill_cache_write(k, v, 7)
    assert kc.dtype == k.dtype and (kc[:, :, 3:] == 0).all() and (vc[:, :, 3:] == 0).all()
    assert np.array_equal(kc[:, :, :3], np.stack([k[:, :, g] for g in range(2)], axis=1))


def test_bf16_bits_are_copied_unchanged():
    k = synth.normal((1, 5, 2, 8), synth.BF16, 43, 2)
    v = synth.normal((1, 5, 2, 8), synth.BF16, 43, 3)
    kc0 = np.full((1, 2, 6, 8), 0x7FC0, dtype=np.uint16)  # NaN sentinel rows
    kc, vc = oracle.prefill_cache_write(k, v, 6, kc0, kc0)
    assert kc.dtype == np.uint16
    for g in range(2):
        assert np.array_equal(kc[0, g, :5], k[0, :, g]) and np.array_equal(vc[0, g, :5], v[0, :, g])
    assert (kc[0, :, 5] == 0x7FC0).all()


def test_equal_lengths_match_the_varlen_form():
    B, S, K, d, S_max = 3, 6, 2, 4, 8
    k, v = rnd((B, S, K, d), 44, 2), rnd((B, S, K, d), 44, 3)
    kc0 = np.full((B, K, S_max, d), 1.5)
    vc0 = np.full((B, K, S_max, d), -1.5)
    fixed = oracle.prefill_cache_write(k, v, S_max, kc0, vc0)
    cu = np.arange(B + 1, dtype=np.int32) * S
    packed = oracle.prefill_cache_write_varlen(k.reshape(B * S, K, d), v.reshape(B * S, K, d), cu, S_max, kc0, vc0)
    assert np.array_equal(fixed[0], packed[0]) and np.array_equal(fixed[1], packed[1])


# ---------------------------------------------------------------------------
# planted mistakes: each must fail the loop check


def _mut_axes_kept(k, v, S_max, k_cache, v_cache):  # the token and head axes not swapped
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    S = k.shape[1]
    kc[:, :, :S, :] = k
    vc[:, :, :S, :] = v
    return kc, vc


def _mut_k_for_v(k, v, S_max, k_cache, v_cache):  # K's rows written to both caches
    return oracle.prefill_cache_write(k, k, S_max, k_cache, v_cache)


def _mut_row_offset(k, v, S_max, k_cache, v_cache):  # token t written at key t + 1
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    S = k.shape[1]
    kc[:, :, 1:S + 1, :] = np.transpose(k, (0, 2, 1, 3))
    vc[:, :, 1:S + 1, :] = np.transpose(v, (0, 2, 1, 3))
    return kc, vc


def _mut_whole_cache(k, v, S_max, k_cache, v_cache):  # rows past the prompt cleared
    kc, vc = oracle.prefill_cache_write(k, v, S_max, k_cache, v_cache)
    S = k.shape[1]
    kc[:, :, S:] = 0
    vc[:, :, S:] = 0
    return kc, vc


def test_planted_cache_write_mistakes_are_caught():
    assert _loop_check(oracle.prefill_cache_write)
    for mutant in (_mut_axes_kept, _mut_k_for_v, _mut_row_offset, _mut_whole_cache):
        assert not _loop_check(mutant), mutant.__name__
