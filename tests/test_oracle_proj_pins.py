"""Pins for the oracle's fused K/V projection into the cache.

The reading ("GQA 完全拆解", section 工程实现：权重布局、repeat 与 Kernel 融合:
one merged W_KV [K, 2 d_k, d_model], one GEMM for K and V): for KV head g,
W_KV[g] x gives 2d values, K's d then V's, written at the token's key.

Checked by brute force on tiny inputs, a one-hot weight whose outputs are
known entries of x (head, K/V half and row order in one), linearity, a
weight with zero V rows, and the cache placement; planted mistakes in the
projection (swapped halves, the neighbouring head's weights, a transposed
weight) each fail.
"""
import numpy as np

import oracle
import synth


def rnd(shape, seed, stream):
    return synth.normal(shape, synth.F64, seed, stream)


def check_brute_force(proj):
    x, w = rnd((2, 3, 12), 51, 1), rnd((2, 8, 12), 51, 2)  # B 2, T 3, d_model 12; K 2, d 4
    got = proj(x, w)
    for b in range(2):
        for t in range(3):
            for g in range(2):
                for j in range(8):
                    acc = 0.0
                    for c in range(12):
                        acc += w[g, j, c] * x[b, t, c]
                    if abs(got[b, t, g, j] - acc) > 1e-12:
                        return False
    return True


def check_one_hot(proj):
    K, d, dm = 3, 4, 32
    w = np.zeros((K, 2 * d, dm))
    for g in range(K):
        for j in range(2 * d):
            w[g, j, (g * 2 * d + j) % dm] = 1.0
    x = rnd((5, dm), 52, 1)
    got = proj(x, w)
    for g in range(K):
        for j in range(2 * d):
            if not np.array_equal(got[:, g, j], x[:, (g * 2 * d + j) % dm]):
                return False
    return True


def check_linear_and_halves(proj):
    x1, x2, w = rnd((4, 16), 53, 1), rnd((4, 16), 53, 2), rnd((2, 6, 16), 53, 3)
    if np.max(np.abs(proj(x1 + x2, w) - proj(x1, w) - proj(x2, w))) > 1e-12:
        return False
    w0 = w.copy()
    w0[:, 3:, :] = 0.0  # zero V rows (d = 3): V outputs zero, K outputs unchanged
    a, b = proj(x1, w0), proj(x1, w)
    return np.all(a[..., 3:] == 0) and np.array_equal(a[..., :3], b[..., :3])


CHECKS = [check_brute_force, check_one_hot, check_linear_and_halves]


def test_projection_pins():
    for check in CHECKS:
        assert check(oracle.kv_project), check.__name__


def test_append_places_rows():
    B, T, K, d, dm, S_max = 3, 2, 2, 4, 16, 6
    x, w = rnd((B, T, dm), 54, 1), rnd((K, 2 * d, dm), 54, 2)
    kc0 = np.full((B, K, S_max, d), -5.0)
    pos = np.array([0, 4, 5], np.int32)  # the last one does not fit (5 + 2 > 6)
    kc, vc = oracle.kv_project_append(kc0, kc0, x, w, pos, like_dtype=np.float64)
    kv = oracle.kv_project(x, w)
    for b in range(2):
        for i in range(T):
            assert np.array_equal(kc[b, :, pos[b] + i], kv[b, i, :, :d])
            assert np.array_equal(vc[b, :, pos[b] + i], kv[b, i, :, d:])
    assert (kc[2] == -5.0).all() and (kc[0, :, 2:] == -5.0).all() and (kc[1, :, :4] == -5.0).all()


# planted mistakes
def _mut_swapped_halves(x, w):
    out = oracle.kv_project(x, w)
    d = w.shape[1] // 2
    return np.concatenate([out[..., d:], out[..., :d]], axis=-1)


def _mut_next_head(x, w):
    return oracle.kv_project(x, np.roll(np.asarray(w), 1, axis=0))


def _mut_transposed(x, w):
    K, two_d, dm = w.shape
    wt = np.asarray(w).reshape(K * two_d, dm).T.reshape(dm, K * two_d)  # [d_model, K*2d] read as rows
    if dm != K * two_d:
        wt = np.resize(wt, (K * two_d, dm))
    return oracle.kv_project(x, wt.reshape(K, two_d, dm))


def test_planted_projection_mistakes_are_caught():
    for mutant in (_mut_swapped_halves, _mut_next_head, _mut_transposed):
        assert not all(check(mutant) for check in CHECKS), mutant.__name__
