"""Pins for the oracle's paged decode attention (CPU only).

The oracle must equal ordinary attention over the concatenated tokens.  It is
checked against: torch's CPU scaled_dot_product_attention in float64 on K/V
built contiguously without any block table (a library routine), closed forms
(one token, two tokens, equal keys, zero scale), a 40-digit mpmath evaluation
for large scores, and invariances (block-id relabelling, shared prefix vs a
private copy).
"""

import math

import mpmath
import numpy as np
import pytest
import torch

from oracle import OraclePool, gather_kv, oracle_decode, oracle_decode_one


def scatter_sequences(rng, num_blocks, bs, hkv, d, lens, order=None):
    """Random logical K/V per sequence, written into a pool through fresh tables.

    Returns (k_pool, v_pool, tables, logical_k, logical_v).  Unused pool
    entries hold NaN so any stray read shows up.
    """
    pool = OraclePool(num_blocks, bs, order)
    kp = np.full((num_blocks, bs, hkv, d), np.nan)
    vp = np.full((num_blocks, bs, hkv, d), np.nan)
    tables, lk, lv = [], [], []
    for n in lens:
        t = []
        k = rng.standard_normal((n, hkv, d))
        v = rng.standard_normal((n, hkv, d))
        length = 0
        for j in range(n):
            slot, length, _, _ = pool.reserve_slot(t, length)
            kp[slot // bs, slot % bs] = k[j]
            vp[slot // bs, slot % bs] = v[j]
        tables.append(t)
        lk.append(k)
        lv.append(v)
    return kp, vp, tables, lk, lv


def sdpa(q_sh, k, v, scale):
    """torch float64 scaled_dot_product_attention for one sequence; q [Hq, D], k/v [n, Hkv, D]."""
    qt = torch.from_numpy(q_sh)[None, :, None, :]
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)
    return out[0, :, 0, :].numpy()


@pytest.mark.parametrize("hq,hkv,bs", [(2, 2, 16), (8, 2, 4), (4, 1, 8), (6, 3, 1)])
def test_matches_library_attention(hq, hkv, bs):
    rng = np.random.default_rng(hq * 100 + hkv * 10 + bs)
    d = 16
    lens = [1, bs, bs + 1, 3 * bs + 5, 7]
    nb = sum(-(-n // bs) for n in lens) + 3
    order = rng.permutation(nb)
    kp, vp, tables, lk, lv = scatter_sequences(rng, nb, bs, hkv, d, lens, order)
    q = rng.standard_normal((len(lens), hq, d))
    scale = 1.0 / math.sqrt(d)
    out = oracle_decode(q, kp, vp, tables, lens, scale)
    for s in range(len(lens)):
        ref = sdpa(q[s], lk[s], lv[s], scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_gather_returns_tokens_in_logical_order():
    rng = np.random.default_rng(5)
    kp, vp, tables, lk, lv = scatter_sequences(rng, 12, 4, 2, 3, [10, 1], rng.permutation(12))
    for s, n in enumerate([10, 1]):
        k, v = gather_kv(kp, vp, tables[s], n, 4)
        assert np.array_equal(k, lk[s]) and np.array_equal(v, lv[s])


def test_block_relabelling_is_bit_invariant():
    rng = np.random.default_rng(11)
    nb, bs, hkv, d = 20, 4, 2, 8
    lens = [13, 4, 1, 9]
    kp, vp, tables, _, _ = scatter_sequences(rng, nb, bs, hkv, d, lens)
    q = rng.standard_normal((len(lens), 4, d))
    base = oracle_decode(q, kp, vp, tables, lens, 0.3)
    perm = rng.permutation(nb)                        # physical id b -> perm[b]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    tables2 = [[int(perm[b]) for b in t] for t in tables]
    moved = oracle_decode(q, kp2, vp2, tables2, lens, 0.3)
    assert np.array_equal(base, moved)


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(2)
    for _ in range(20):
        q = rng.standard_normal(32) * 10
        k = rng.standard_normal((1, 32))
        v = rng.standard_normal((1, 32))
        assert np.array_equal(oracle_decode_one(q, k, v, 0.7), v[0])


def test_two_tokens_closed_form():
    # softmax over two scores is the logistic function of their difference
    rng = np.random.default_rng(3)
    for _ in range(20):
        q = rng.standard_normal(16)
        k = rng.standard_normal((2, 16))
        v = rng.standard_normal((2, 16))
        scale = rng.uniform(0.05, 1.0)
        w1 = 1.0 / (1.0 + math.exp(-scale * float(q @ (k[1] - k[0]))))
        expect = v[0] + w1 * (v[1] - v[0])
        np.testing.assert_allclose(oracle_decode_one(q, k, v, scale), expect, rtol=0, atol=1e-13)


def test_equal_keys_and_zero_scale_give_mean_of_values():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((37, 8))
    q = rng.standard_normal(8)
    same = np.tile(rng.standard_normal(8), (37, 1))
    np.testing.assert_allclose(oracle_decode_one(q, same, v, 0.5), v.mean(0), rtol=0, atol=1e-12)
    k = rng.standard_normal((37, 8))
    np.testing.assert_allclose(oracle_decode_one(q, k, v, 0.0), v.mean(0), rtol=0, atol=1e-12)


def test_large_scores_match_high_precision():
    rng = np.random.default_rng(6)
    mpmath.mp.dps = 40
    q = rng.standard_normal(16) * 30
    k = rng.standard_normal((50, 16))
    v = rng.standard_normal((50, 16))
    out = oracle_decode_one(q, k, v, 0.25)
    assert np.all(np.isfinite(out))
    scores = [mpmath.mpf(float(x)) for x in (k @ q)]
    w = [mpmath.e ** (mpmath.mpf(0.25) * s) for s in scores]
    total = mpmath.fsum(w)
    for dcol in range(16):
        ref = mpmath.fsum(w[j] * mpmath.mpf(float(v[j, dcol])) for j in range(50)) / total
        assert abs(float(ref) - out[dcol]) <= 1e-12 * max(1.0, abs(float(ref)))


def test_shared_prefix_equals_private_copy():
    rng = np.random.default_rng(8)
    nb, bs, hkv, d = 40, 4, 2, 8
    pool = OraclePool(nb, bs)
    kp = rng.standard_normal((nb, bs, hkv, d))
    vp = rng.standard_normal((nb, bs, hkv, d))
    prefix = pool.alloc(3)                             # 12 shared tokens
    shared = [prefix + pool.alloc(2), prefix + pool.alloc(1)]
    lens = [19, 14]
    # private copies: duplicate the prefix blocks into fresh blocks
    copies = pool.alloc(6)
    private = [copies[:3] + shared[0][3:], copies[3:] + shared[1][3:]]
    kp[copies[:3]] = kp[prefix]
    vp[copies[:3]] = vp[prefix]
    kp[copies[3:]] = kp[prefix]
    vp[copies[3:]] = vp[prefix]
    q = rng.standard_normal((2, 4, d))
    a = oracle_decode(q, kp, vp, shared, lens, 0.35)
    b = oracle_decode(q, kp, vp, private, lens, 0.35)
    assert np.array_equal(a, b)


def test_grouped_heads_equal_repeated_kv_heads():
    rng = np.random.default_rng(9)
    nb, bs, d = 10, 4, 8
    lens = [11, 5]
    kp, vp, tables, _, _ = scatter_sequences(rng, nb, bs, 2, d, lens)
    q = rng.standard_normal((2, 6, d))
    grouped = oracle_decode(q, kp, vp, tables, lens, 0.4)
    rep_k = np.repeat(kp, 3, axis=2)                   # KV head j serves query heads 3j..3j+2
    rep_v = np.repeat(vp, 3, axis=2)
    mha = oracle_decode(q, rep_k, rep_v, tables, lens, 0.4)
    assert np.array_equal(grouped, mha)


def test_zero_length_gives_zero_row():
    kp = np.ones((2, 4, 1, 3))
    out = oracle_decode(np.ones((1, 2, 3)), kp, kp, [[0]], [0], 1.0)
    assert np.array_equal(out, np.zeros((1, 2, 3)))
