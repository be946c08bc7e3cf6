"""Pins for the oracle's host block pool (CPU only).

Each test fixes the oracle to something other than itself: the worked example
printed on the agentechip page, the memory claim on the aidolsgroup page, and
invariants that any correct pool must keep.
"""

import random

import pytest

from oracle import OraclePool, PoolExhausted, RefcountError, InvalidRequest
from golden_io import read_golden


def grow(pool, table, length, n):
    """Reserve ``n`` more slots for one sequence; returns (slots, length, cow pairs)."""
    slots, pairs = [], []
    for _ in range(n):
        slot, length, src, dst = pool.reserve_slot(table, length)
        slots.append(slot)
        if src >= 0:
            pairs.append((src, dst))
    return slots, length, pairs


def test_toy_worked_example():
    g = read_golden("toy_worked_example.txt")
    pool = OraclePool(g["num_blocks"], g["block_size"])
    table, length = [], 0
    slots, length, pairs = grow(pool, table, length, g["tokens_appended"])
    assert length == g["tokens_cached"]
    assert len(table) == g["blocks_used"]
    per_block = [sum(1 for s in slots if s // g["block_size"] == b) for b in table]
    assert per_block == g["tokens_per_block"]
    assert pairs == []
    pool.free(table)
    assert pool.num_free() == g["free_blocks_after_free"]


def test_blocks_needed_is_ceiling_of_length():
    for bs in (1, 8, 16, 32):
        for n in range(0, 100):
            pool = OraclePool(200, bs)
            table = []
            grow(pool, table, 0, n)
            assert len(table) == -(-n // bs)
            assert pool.num_free() == 200 - len(table)


def test_free_list_is_first_in_first_out():
    pool = OraclePool(6, 4)
    assert pool.alloc(3) == [0, 1, 2]
    pool.free([1])
    pool.free([0])
    # front of the list is still 3, 4, 5; released blocks queue behind them
    assert pool.alloc(5) == [3, 4, 5, 1, 0]
    assert pool.num_free() == 0 and pool.refcount(2) == 1


def test_initial_order_is_respected():
    order = [5, 2, 7, 0, 1, 3, 6, 4]
    pool = OraclePool(8, 16, order)
    assert pool.alloc(8) == order
    with pytest.raises(InvalidRequest):
        OraclePool(3, 16, [0, 0, 1])


def test_exhaustion_changes_nothing():
    pool = OraclePool(4, 2, [3, 1, 0, 2])
    table, length = [], 0
    _, length, _ = grow(pool, table, length, 8)       # all 4 blocks full
    before = pool.export(), list(table), length
    with pytest.raises(PoolExhausted):
        pool.reserve_slot(table, length)
    assert (pool.export(), table, length) == before
    with pytest.raises(PoolExhausted):
        pool.alloc(1)
    assert pool.export() == before[0]


def test_copy_on_write_only_for_shared_partial_block():
    pool = OraclePool(10, 4)
    parent, plen = [], 0
    _, plen, _ = grow(pool, parent, plen, 6)            # blocks [0, 1], last one half full
    pool.fork(parent)
    child, clen = list(parent), plen
    assert [pool.refcount(b) for b in parent] == [2, 2]
    slot, clen, src, dst = pool.reserve_slot(child, clen)
    assert (src, dst) == (1, 2)                        # shared block 1 moves to fresh block 2
    assert child == [0, 2] and slot == 2 * 4 + 2
    assert pool.refcount(1) == 1 and pool.refcount(2) == 1 and pool.refcount(0) == 2
    # the parent now owns block 1 alone: no further copy
    slot, plen, src, dst = pool.reserve_slot(parent, plen)
    assert (src, dst) == (-1, -1) and slot == 1 * 4 + 2
    # a shared full block: the next token opens a fresh block, nothing copied
    pool2 = OraclePool(10, 4)
    p2, l2 = [], 0
    _, l2, _ = grow(pool2, p2, l2, 8)
    pool2.fork(p2)
    c2 = list(p2)
    slot, l2c, src, dst = pool2.reserve_slot(c2, l2)
    assert (src, dst) == (-1, -1) and c2[:2] == p2 and len(c2) == 3


def test_copy_on_write_exhaustion_changes_nothing():
    pool = OraclePool(2, 4)
    parent, plen = [], 0
    _, plen, _ = grow(pool, parent, plen, 3)
    pool.fork(parent)
    pool.alloc(1)                                      # last free block gone
    child = list(parent)
    before = pool.export(), list(child)
    with pytest.raises(PoolExhausted):
        pool.reserve_slot(child, plen)
    assert (pool.export(), child) == before


def test_refcount_errors_change_nothing():
    pool = OraclePool(4, 4)
    ids = pool.alloc(2)
    before = pool.export()
    with pytest.raises(RefcountError):
        pool.free([ids[0], ids[0]])                    # only one reference held
    with pytest.raises(RefcountError):
        pool.fork([3])                                 # block 3 is free
    with pytest.raises(InvalidRequest):
        pool.free([9])
    assert pool.export() == before


def test_invariants_under_random_scripts():
    rng = random.Random(341)
    for trial in range(40):
        nb, bs = rng.randint(1, 24), rng.choice([1, 2, 4, 16])
        order = list(range(nb))
        rng.shuffle(order)
        pool = OraclePool(nb, bs, order)
        seqs = {}                                      # id -> [table, length]
        next_id = 0
        for _ in range(200):
            op = rng.random()
            try:
                if op < 0.55 and seqs:
                    sid = rng.choice(list(seqs))
                    t, n = seqs[sid]
                    _, n, _, _ = pool.reserve_slot(t, n)
                    seqs[sid][1] = n
                elif op < 0.7:
                    seqs[next_id] = [[], 0]
                    next_id += 1
                elif op < 0.85 and seqs:
                    sid = rng.choice(list(seqs))
                    t, n = seqs[sid]
                    pool.fork(t)
                    seqs[next_id] = [list(t), n]
                    next_id += 1
                elif seqs:
                    sid = rng.choice(list(seqs))
                    pool.free(seqs.pop(sid)[0])
            except PoolExhausted:
                pass
            refs, free = pool.export()
            held = [b for t, _ in seqs.values() for b in t]
            assert sum(refs) == len(held)
            for b in range(nb):
                assert refs[b] == held.count(b)
            assert len(free) == len(set(free))
            assert set(free) == {b for b in range(nb) if refs[b] == 0}
            for t, n in seqs.values():
                assert len(t) == -(-n // bs)


def test_shared_prompt_frees_at_least_the_claimed_fraction():
    g = read_golden("shared_prompt_example.txt")
    bs, users = g["block_size"], g["users"]
    prefix_blocks = g["prefix_tokens"] // bs
    rng = random.Random(7)
    suffixes = [rng.randint(1, 512) for _ in range(users)]
    pool = OraclePool(prefix_blocks + sum(-(-s // bs) for s in suffixes) + 8, bs)
    prefix, plen = [], 0
    _, plen, _ = grow(pool, prefix, plen, g["prefix_tokens"])
    tables = []
    for s in suffixes:
        pool.fork(prefix)
        t, n = list(prefix), plen
        _, n, pairs = grow(pool, t, n, s)
        assert pairs == []                               # the prefix ends on a block boundary
        tables.append(t)
    pool.free(prefix)                                    # the prompt owner leaves
    shared_used = pool.num_blocks - pool.num_free()
    unshared_used = sum(len(t) for t in tables)
    freed = 1.0 - shared_used / unshared_used
    assert freed >= g["claimed_fraction_freed_at_least"]
    assert pool.refcount(prefix[0]) == users
