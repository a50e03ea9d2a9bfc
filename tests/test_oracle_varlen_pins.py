"""Pins for the oracle's varlen (packed) causal prefill.

Each sequence of a packed batch is prefilled causally on its own. Checked
against torch's float64 causal scaled_dot_product_attention run sequence by
sequence on the test's own slices, against the oracle's fixed-length prefill
when every sequence has the same length (the [B, S] layout), and by
isolation: changing one sequence's tokens leaves every other sequence's
output unchanged. The cache write places row t of sequence b at key t.
"""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
import synth


def rnd(shape, seed, stream):
    return synth.normal(shape, synth.F64, seed, stream)


def test_varlen_vs_torch_per_sequence():
    lens = [5, 1, 12, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, K, d = int(cu[-1]), 6, 2, 16
    q, k, v = rnd((T, H, d), 31, 1), rnd((T, K, d), 31, 2), rnd((T, K, d), 31, 3)
    got = oracle.prefill_causal_varlen(q, k, v, cu, 0.3)
    for b, n in enumerate(lens):
        s = slice(cu[b], cu[b + 1])
        qt = torch.from_numpy(np.ascontiguousarray(np.transpose(q[s], (1, 0, 2))))[None]
        kt = torch.from_numpy(np.ascontiguousarray(np.transpose(k[s], (1, 0, 2))))[None]
        vt = torch.from_numpy(np.ascontiguousarray(np.transpose(v[s], (1, 0, 2))))[None]
        want = F.scaled_dot_product_attention(qt, kt, vt, scale=0.3, is_causal=True, enable_gqa=True)[0]
        assert np.max(np.abs(got[s] - np.transpose(want.numpy(), (1, 0, 2)))) < 1e-12


def test_equal_lengths_match_the_fixed_length_prefill():
    B, S, H, K, d = 3, 9, 4, 2, 8
    q, k, v = rnd((B, S, H, d), 32, 1), rnd((B, S, K, d), 32, 2), rnd((B, S, K, d), 32, 3)
    cu = np.arange(B + 1, dtype=np.int32) * S
    got = oracle.prefill_causal_varlen(q.reshape(B * S, H, d), k.reshape(B * S, K, d), v.reshape(B * S, K, d), cu, 0.2)
    want = oracle.prefill_causal(q, k, v, 0.2).reshape(B * S, H, d)
    assert np.array_equal(got, want)


def test_sequences_are_isolated():
    lens = [6, 4, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, K, d = int(cu[-1]), 4, 1, 8
    q, k, v = rnd((T, H, d), 33, 1), rnd((T, K, d), 33, 2), rnd((T, K, d), 33, 3)
    base = oracle.prefill_causal_varlen(q, k, v, cu, 0.25)
    k2, v2 = k.copy(), v.copy()
    k2[cu[1]:cu[2]] += 1.0
    v2[cu[1]:cu[2]] -= 2.0
    pert = oracle.prefill_causal_varlen(q, k2, v2, cu, 0.25)
    assert np.array_equal(pert[:cu[1]], base[:cu[1]]) and np.array_equal(pert[cu[2]:], base[cu[2]:])
    assert np.max(np.abs(pert[cu[1]:cu[2]] - base[cu[1]:cu[2]])) > 1e-3
    # first token of every sequence: its own value row
    for b in range(3):
        assert np.allclose(base[cu[b]], v[cu[b], 0][None, :].repeat(H, 0), atol=1e-15)


def test_varlen_cache_write_rows():
    lens = [3, 0, 5]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, K, d, S_max = int(cu[-1]), 2, 4, 6
    k, v = rnd((T, K, d), 34, 2), rnd((T, K, d), 34, 3)
    kc0 = np.full((3, K, S_max, d), -7.0)
    kc, vc = oracle.prefill_cache_write_varlen(k, v, cu, S_max, kc0, kc0)
    for b in range(3):
        for t in range(lens[b]):
            assert np.array_equal(kc[b, :, t], k[cu[b] + t]) and np.array_equal(vc[b, :, t], v[cu[b] + t])
        assert (kc[b, :, lens[b]:] == -7.0).all()


def test_varlen_workload_lengths():
    w = synth.VARLEN_WORKLOADS["varlen_prefill_b8_h32_k8_d128_s256_4k"]
    lens = synth.uniform_int(w.B, w.len_range[0], w.len_range[1], w.seed, synth.STREAM_LENS)
    assert lens.min() >= 256 and lens.max() <= 4096 and lens.max() <= w.S_max


# ---------------------------------------------------------------------------
# planted mistakes in the varlen decomposition: each must fail a check

def _check_torch(impl):
    lens = [5, 1, 12, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, K, d = int(cu[-1]), 6, 2, 16
    q, k, v = rnd((T, H, d), 35, 1), rnd((T, K, d), 35, 2), rnd((T, K, d), 35, 3)
    got = impl(q, k, v, cu, 0.3)
    for b in range(len(lens)):
        s = slice(cu[b], cu[b + 1])
        qt = torch.from_numpy(np.ascontiguousarray(np.transpose(q[s], (1, 0, 2))))[None]
        kt = torch.from_numpy(np.ascontiguousarray(np.transpose(k[s], (1, 0, 2))))[None]
        vt = torch.from_numpy(np.ascontiguousarray(np.transpose(v[s], (1, 0, 2))))[None]
        want = F.scaled_dot_product_attention(qt, kt, vt, scale=0.3, is_causal=True, enable_gqa=True)[0]
        if np.max(np.abs(got[s] - np.transpose(want.numpy(), (1, 0, 2)))) > 1e-12:
            return False
    return True


def _mut_one_sequence(q, k, v, cu, scale):  # attends across sequence boundaries
    return oracle.prefill_causal(q[None], k[None], v[None], scale)[0]


def _mut_boundary_off_by_one(q, k, v, cu, scale):  # sequence b starts one token late
    cu2 = np.array(cu).copy()
    cu2[1:-1] += 1
    return oracle.prefill_causal_varlen(q, k, v, cu2, scale)


def test_planted_varlen_mistakes_are_caught():
    assert _check_torch(oracle.prefill_causal_varlen)
    for mutant in (_mut_one_sequence, _mut_boundary_off_by_one):
        assert not _check_torch(mutant), mutant.__name__
