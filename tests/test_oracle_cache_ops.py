"""Pins for the oracle's append and block copy (CPU only)."""

import hashlib

import numpy as np

from oracle import OraclePool, gather_kv, oracle_append, oracle_copy_blocks


def digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def test_append_places_token_at_end_of_sequence():
    rng = np.random.default_rng(1)
    nb, bs, hkv, d = 8, 4, 2, 3
    pool = OraclePool(nb, bs, rng.permutation(nb))
    kc = rng.standard_normal((nb, bs, hkv, d))
    vc = rng.standard_normal((nb, bs, hkv, d))
    table, length = [], 0
    rows_k, rows_v = [], []
    for step in range(11):
        slot, length, _, _ = pool.reserve_slot(table, length)
        kn = rng.standard_normal((1, hkv, d))
        vn = rng.standard_normal((1, hkv, d))
        oracle_append(kc, vc, kn, vn, [slot])
        rows_k.append(kn[0])
        rows_v.append(vn[0])
        k, v = gather_kv(kc, vc, table, length, bs)
        assert np.array_equal(k, np.stack(rows_k)) and np.array_equal(v, np.stack(rows_v))


def test_append_touches_only_its_slots_and_skips_negative():
    rng = np.random.default_rng(2)
    kc = rng.integers(0, 1 << 16, (6, 4, 2, 5)).astype(np.uint16)
    vc = rng.integers(0, 1 << 16, (6, 4, 2, 5)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    kn = rng.integers(0, 1 << 16, (3, 2, 5)).astype(np.uint16)
    vn = rng.integers(0, 1 << 16, (3, 2, 5)).astype(np.uint16)
    oracle_append(kc, vc, kn, vn, [13, -1, 0])
    assert np.array_equal(kc[3, 1], kn[0]) and np.array_equal(vc[0, 0], vn[2])
    kc[3, 1], vc[3, 1] = k0[3, 1], v0[3, 1]
    kc[0, 0], vc[0, 0] = k0[0, 0], v0[0, 0]
    assert digest(kc) == digest(k0) and digest(vc) == digest(v0)


def test_copy_blocks_duplicates_whole_blocks_only():
    rng = np.random.default_rng(3)
    kc = rng.integers(0, 1 << 16, (7, 4, 2, 5)).astype(np.uint16)
    vc = rng.integers(0, 1 << 16, (7, 4, 2, 5)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    oracle_copy_blocks(kc, vc, [(1, 4), (6, 0)])
    assert np.array_equal(kc[4], k0[1]) and np.array_equal(vc[4], v0[1])
    assert np.array_equal(kc[0], k0[6]) and np.array_equal(vc[0], v0[6])
    for b in (1, 2, 3, 5, 6):
        assert np.array_equal(kc[b], k0[b]) and np.array_equal(vc[b], v0[b])


def test_copy_on_write_keeps_both_sequences_intact():
    rng = np.random.default_rng(4)
    nb, bs = 10, 4
    pool = OraclePool(nb, bs)
    kc = np.zeros((nb, bs, 1, 2))
    vc = np.zeros((nb, bs, 1, 2))
    parent, plen = [], 0
    for _ in range(6):
        slot, plen, _, _ = pool.reserve_slot(parent, plen)
        oracle_append(kc, vc, rng.standard_normal((1, 1, 2)), rng.standard_normal((1, 1, 2)), [slot])
    before = gather_kv(kc, vc, parent, plen, bs)
    pool.fork(parent)
    child, clen = list(parent), plen
    slot, clen, src, dst = pool.reserve_slot(child, clen)
    oracle_copy_blocks(kc, vc, [(src, dst)])
    new_k, new_v = rng.standard_normal((1, 1, 2)), rng.standard_normal((1, 1, 2))
    oracle_append(kc, vc, new_k, new_v, [slot])
    after_parent = gather_kv(kc, vc, parent, plen, bs)
    ck, cv = gather_kv(kc, vc, child, clen, bs)
    assert np.array_equal(after_parent[0], before[0]) and np.array_equal(after_parent[1], before[1])
    assert np.array_equal(ck[:plen], before[0]) and np.array_equal(ck[plen], new_k[0])
    assert np.array_equal(cv[:plen], before[1]) and np.array_equal(cv[plen], new_v[0])
