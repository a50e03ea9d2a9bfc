"""Pins for the oracle's paged KV cache (block table over a pool of blocks).

The reading (the pages give no block size or table format): a pool
[num_blocks, K, block_size, d] and a table [B, max_blocks] whose entry
(b, i) is the physical block holding keys i*block_size .. (i+1)*block_size-1
of sequence b, for every KV head of the group ("分組查詢注意力", section
下游 / 推論引擎與架構; "GQA 完全拆解", section 工程实现：权重布局、repeat 与 Kernel 融合).

Each pin ties the paged oracle to something other than itself: torch's
float64 scaled_dot_product_attention on the contiguous cache the pool was
scattered from (the scatter here is written independently, with torch
indexing), invariance under moving blocks, blocks that must never be read,
and the two degenerate block sizes. The last test runs the same pins on
planted mistakes in the gather and shows that each one fails.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def rnd(shape, seed, stream):
    return synth.normal(shape, synth.F64, seed, stream)


def sdpa_decode(q, kc, vc, lens, scale):
    B, H, d = q.shape
    out = np.zeros((B, H, d))
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        qt = torch.from_numpy(q[b][None, :, None, :])
        kt = torch.from_numpy(np.ascontiguousarray(kc[b][None, :, :n, :]))
        vt = torch.from_numpy(np.ascontiguousarray(vc[b][None, :, :n, :]))
        out[b] = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)[0, :, 0, :].numpy()
    return out


def scatter(cache, lens, bs, order, spare=3):
    """Independent scatter (torch indexing): blocks of sequence b go to pool slots taken in `order`."""
    B, K, S, d = cache.shape
    mb = S // bs
    need = [(int(n) + bs - 1) // bs for n in lens]
    nb = sum(need) + spare
    pool = torch.full((nb, K, bs, d), float("nan"), dtype=torch.float64)
    table = torch.full((B, mb), -1, dtype=torch.int32)
    c = torch.from_numpy(cache)
    slots = iter([int(o) for o in order if o < nb])  # the order restricted to the pool's slots
    for b in range(B):
        for i in range(need[b]):
            blk = next(slots)
            table[b, i] = blk
            pool[blk] = c[b, :, i * bs:(i + 1) * bs, :]
    return pool.numpy(), table.numpy()


SHAPES = [
    # B, H, K, d, S_max, block_size, lens
    (2, 8, 2, 16, 32, 8, (32, 13)),
    (3, 6, 1, 8, 24, 4, (24, 1, 9)),      # MQA
    (2, 4, 4, 8, 16, 16, (16, 7)),        # MHA; one block per sequence
    (1, 12, 3, 32, 20, 1, (17,)),         # every key its own block
]


def decode_paged_with(gather, q, kp, vp, table, lens, scale):
    return oracle.decode(q, gather(kp, table), gather(vp, table), lens, scale)


def check_vs_sdpa(gather):
    for i, (B, H, K, d, S, bs, lens) in enumerate(SHAPES):
        q, kc, vc = rnd((B, H, d), 40 + i, 1), rnd((B, K, S, d), 40 + i, 2), rnd((B, K, S, d), 40 + i, 3)
        lens = np.array(lens, dtype=np.int32)
        order = np.random.default_rng(7 + i).permutation(64)
        kp, table = scatter(kc, lens, bs, order)
        vp, _ = scatter(vc, lens, bs, order)
        scale = 1.0 / np.sqrt(d)
        got = decode_paged_with(gather, q, kp, vp, table, lens, scale)
        want = sdpa_decode(q, kc, vc, lens, scale)
        if not np.all(np.isfinite(got)) or np.max(np.abs(got - want)) > 1e-12:
            return False
    return True


def check_block_moves(gather):
    B, H, K, d, S, bs = 2, 8, 2, 16, 48, 8
    lens = np.array([48, 30], dtype=np.int32)
    q, kc, vc = rnd((B, H, d), 60, 1), rnd((B, K, S, d), 60, 2), rnd((B, K, S, d), 60, 3)
    outs = []
    for seed in (1, 2, 3):
        order = np.random.default_rng(seed).permutation(64)
        kp, table = scatter(kc, lens, bs, order)
        vp, _ = scatter(vc, lens, bs, order)
        outs.append(decode_paged_with(gather, q, kp, vp, table, lens, 0.25))
    return all(np.all(np.isfinite(o)) for o in outs) and all(np.array_equal(outs[0], o) for o in outs[1:])


PAGED_CHECKS = [check_vs_sdpa, check_block_moves]


@pytest.mark.parametrize("check", PAGED_CHECKS, ids=lambda f: f.__name__)
def test_paged_pin(check):
    assert check(oracle.paged_gather)


def test_unreferenced_blocks_are_never_read():
    # -1 table entries past each length and NaN pool blocks: the output stays finite
    B, H, K, d, S, bs = 2, 4, 2, 8, 32, 8
    lens = np.array([9, 25], dtype=np.int32)
    q, kc, vc = rnd((B, H, d), 70, 1), rnd((B, K, S, d), 70, 2), rnd((B, K, S, d), 70, 3)
    kp, table = scatter(kc, lens, bs, np.arange(64), spare=5)
    vp, _ = scatter(vc, lens, bs, np.arange(64), spare=5)
    assert (table[0, 2:] == -1).all() and np.isnan(kp[-1]).all()
    got = oracle.decode_paged(q, kp, vp, table, lens, 0.3)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - sdpa_decode(q, kc, vc, lens, 0.3))) < 1e-12


def test_gather_rebuilds_the_cache_rows():
    # every valid key row of every head comes back bit for bit
    B, K, d, S, bs = 3, 2, 8, 40, 8
    lens = np.array([40, 3, 17], dtype=np.int32)
    kc = rnd((B, K, S, d), 80, 2)
    kp, table = scatter(kc, lens, bs, np.random.default_rng(5).permutation(64))
    got = oracle.paged_gather(kp, table)
    for b in range(B):
        assert np.array_equal(got[b, :, :lens[b]], kc[b, :, :lens[b]])


def test_paged_append_writes_one_row_per_head():
    B, K, d, S, bs = 3, 2, 8, 32, 8
    lens = np.array([5, 16, 31], dtype=np.int32)  # appends at 5 (mid-block), 16 (a block's first row), 31
    kc, vc = rnd((B, K, S, d), 90, 2), rnd((B, K, S, d), 90, 3)
    order = np.random.default_rng(9).permutation(64)
    kp, table = scatter(kc, lens + 1, bs, order)
    vp, _ = scatter(vc, lens + 1, bs, order)
    kn, vn = rnd((B, K, d), 90, 5), rnd((B, K, d), 90, 6)
    kp2, vp2 = oracle.kv_append_paged(kp, vp, kn, vn, table, lens)
    for b in range(B):
        blk, r = table[b, lens[b] // bs], lens[b] % bs
        assert np.array_equal(kp2[blk, :, r], kn[b]) and np.array_equal(vp2[blk, :, r], vn[b])
    changed = [(blk, g, r) for blk, g, r in zip(*np.nonzero(np.any(kp2 != kp, axis=-1) & ~np.isnan(kp).all(-1)))]
    assert len(changed) == B * K
    # out-of-range position or table entry: nothing written
    kp3, _ = oracle.kv_append_paged(kp, vp, kn, vn, table, np.array([-1, S, 3], dtype=np.int32))
    bad = table.copy()
    bad[2, 0] = 10 ** 6
    kp4, _ = oracle.kv_append_paged(kp, vp, kn, vn, bad, np.array([-1, S, 3], dtype=np.int32))
    assert np.array_equal(np.nan_to_num(kp3[np.arange(len(kp)) != table[2, 0]]),
                          np.nan_to_num(kp[np.arange(len(kp)) != table[2, 0]]))
    assert np.array_equal(np.nan_to_num(kp4), np.nan_to_num(kp))


# ---------------------------------------------------------------------------
# planted mistakes in the gather: each must fail a pin

def _mut_reversed_rows(pool, table):
    return oracle.paged_gather(pool[:, :, ::-1, :], table)


def _mut_heads_swapped(pool, table):
    nb, K, bs, d = pool.shape
    if K == 1:
        return oracle.paged_gather(pool[:, :, ::-1, :], table)
    return oracle.paged_gather(pool[:, ::-1, :, :], table)


def _mut_block_off_by_one(pool, table):
    t = np.where(table >= 0, (table + 1) % pool.shape[0], table)
    return oracle.paged_gather(pool, t)


def _mut_row_major_blocks(pool, table):
    # reads block i of sequence b from table[i, b] (a transposed table), where that entry exists
    B, mb = table.shape
    t = np.full_like(table, -1)
    for b in range(B):
        for i in range(mb):
            if i < B and b < mb:
                t[b, i] = table[i, b]
    return oracle.paged_gather(pool, t)


@pytest.mark.parametrize("mutant", [_mut_reversed_rows, _mut_heads_swapped, _mut_block_off_by_one,
                                    _mut_row_major_blocks], ids=lambda f: f.__name__)
def test_planted_gather_mistake_is_caught(mutant):
    assert not all(check(mutant) for check in PAGED_CHECKS)
