"""Pins for the oracle's prefix caching by block content (CPU only)."""

import pytest

from oracle import OraclePool, PoolExhausted, fnv1a64, token_bytes
from golden_io import read_golden


def test_fnv1a64_published_vectors():
    # test vectors published with the FNV-1a definition
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_key_covers_block_and_prefix():
    pool = OraclePool(20, 4)
    pool.enable_prefix_cache()
    tokens = [7, 300, -5, 2 ** 31 - 1, 11, 12, 13, 14, 99]
    table, cached = pool.alloc_prompt(tokens)
    assert cached == 0 and len(table) == 3
    keys = {b: k for b, (k, _) in pool.block_key.items()}
    assert keys[table[0]] == fnv1a64(token_bytes(tokens[:4]))
    assert keys[table[1]] == fnv1a64(token_bytes(tokens[:8]))
    assert table[2] not in keys                      # partial block: never registered
    assert token_bytes([1, 256]) == b"\x01\x00\x00\x00\x00\x01\x00\x00"


def test_identical_and_shared_prompts_reuse_full_blocks():
    pool = OraclePool(30, 4, list(range(29, -1, -1)))
    pool.enable_prefix_cache()
    system = list(range(100, 112))                   # 3 full blocks
    t1, c1 = pool.alloc_prompt(system + [1, 2])
    t2, c2 = pool.alloc_prompt(system + [1, 2])
    t3, c3 = pool.alloc_prompt(system + [5, 6, 7, 8, 9])
    assert c1 == 0 and c2 == 12 and c3 == 12
    assert t2[:3] == t1[:3] and t3[:3] == t1[:3]
    assert t2[3] != t1[3]                            # partial last block is private
    assert [pool.refcount(b) for b in t1[:3]] == [3, 3, 3]


def test_same_block_at_another_position_is_not_shared():
    pool = OraclePool(20, 4)
    pool.enable_prefix_cache()
    a, _ = pool.alloc_prompt([1, 2, 3, 4, 5, 6, 7, 8])
    b, cached = pool.alloc_prompt([5, 6, 7, 8, 1, 2, 3, 4])
    assert cached == 0 and not set(a) & set(b)
    c, cached = pool.alloc_prompt([1, 2, 3, 4, 9, 9, 9, 9])
    assert cached == 4 and c[0] == a[0] and c[1] != a[1]


def test_freed_blocks_leave_the_cache_and_failures_change_nothing():
    pool = OraclePool(6, 2)
    pool.enable_prefix_cache()
    t, _ = pool.alloc_prompt([1, 2, 3, 4])
    pool.free(t)
    assert pool.prefix_cache == {}
    t2, cached = pool.alloc_prompt([1, 2, 3, 4])
    assert cached == 0
    before = pool.export(), dict(pool.prefix_cache)
    with pytest.raises(PoolExhausted):
        pool.alloc_prompt([9] * 12)
    assert (pool.export(), pool.prefix_cache) == before


def test_shared_system_prompt_frees_at_least_the_claimed_fraction():
    g = read_golden("shared_prompt_example.txt")
    bs, users, n = g["block_size"], g["users"], g["prefix_tokens"]
    prompt = [(7 * i + 3) % 32000 for i in range(n)]
    pool = OraclePool(n // bs + users * 2 + 4, bs)
    pool.enable_prefix_cache()
    tables = []
    for u in range(users):
        t, cached = pool.alloc_prompt(prompt + [u, u + 1])
        assert cached == (0 if u == 0 else n)
        tables.append(t)
    used = pool.num_blocks - pool.num_free()
    unshared = sum(len(t) for t in tables)
    assert 1.0 - used / unshared >= g["claimed_fraction_freed_at_least"]
