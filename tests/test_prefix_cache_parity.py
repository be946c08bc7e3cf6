"""The library's prefix cache (C++) against the oracle's: identical prompt
scripts give bit-identical tables, cached-token counts, refcounts and free
lists (CPU only)."""

import random

import numpy as np
import pytest

from oracle import OraclePool, PoolExhausted, fnv1a64, token_bytes


@pytest.fixture(scope="module")
def pa(built_library):
    from paged_kv_cache_341_b200 import pa as mod
    return mod


def test_hash_function_matches(pa):
    rng = random.Random(1)
    for n in (0, 1, 5, 64):
        toks = [rng.randint(-2 ** 31, 2 ** 31 - 1) for _ in range(n)]
        assert pa.pa_prefix_hash(toks) == fnv1a64(token_bytes(toks))
    assert pa.pa_prefix_hash([3, 4], seed=12345) == fnv1a64(token_bytes([3, 4]), 12345)


def test_random_prompt_scripts_match(pa):
    rng = random.Random(341)
    for trial in range(30):
        nb, bs = rng.randint(8, 60), rng.choice([1, 2, 4, 16])
        order = list(range(nb))
        rng.shuffle(order)
        lp, op = pa.Pool(nb, bs, order), OraclePool(nb, bs, order)
        lp.pa_pool_enable_prefix_cache()
        op.enable_prefix_cache()
        systems = [[rng.randint(0, 50) for _ in range(rng.randint(0, 3 * bs + 2))] for _ in range(3)]
        live = []
        for _ in range(80):
            if rng.random() < 0.65 or not live:
                toks = rng.choice(systems) + [rng.randint(0, 50) for _ in range(rng.randint(0, 2 * bs))]
                table = np.full(64, -1, np.int32)
                try:
                    cached = lp.pa_seq_alloc_prompt(toks, table)
                    lib = (list(table[: -(-len(toks) // bs)]), cached)
                except pa.PoolExhausted:
                    lib = "exhausted"
                try:
                    ora = op.alloc_prompt(toks)
                except PoolExhausted:
                    ora = "exhausted"
                assert lib == ora
                if lib != "exhausted":
                    live.append(lib[0])
            else:
                t = live.pop(rng.randrange(len(live)))
                lp.pa_pool_free(t)
                op.free(t)
            refs, free = lp.pa_pool_export()
            orefs, ofree = op.export()
            assert list(refs) == orefs and list(free) == ofree
            assert lp.pa_pool_cached_blocks() == len(op.prefix_cache)
