"""The library's host pool (C++) against the oracle pool: identical scripts
give bit-identical block tables, slots, copy pairs, refcounts, free lists and
errors (CPU only)."""

import random

import numpy as np
import pytest

from oracle import OraclePool, PoolExhausted, RefcountError, InvalidRequest
from paged_kv_cache_341_b200 import workloads


@pytest.fixture(scope="module")
def pa(built_library):
    from paged_kv_cache_341_b200 import pa as mod
    return mod


def state_equal(lib_pool, ora_pool):
    refs, free = lib_pool.pa_pool_export()
    orefs, ofree = ora_pool.export()
    return list(refs) == orefs and list(free) == ofree


def test_toy_example_matches(pa):
    lp = pa.Pool(100, 16)
    op = OraclePool(100, 16)
    table = np.full(8, -1, np.int32)
    otable, n, on = [], 0, 0
    for _ in range(40):
        slot, n, src, dst = lp.pa_seq_reserve_slot(table, n)
        oslot, on, osrc, odst = op.reserve_slot(otable, on)
        assert (slot, n, src, dst) == (oslot, on, osrc, odst)
    assert list(table[:3]) == otable and state_equal(lp, op)
    lp.pa_pool_free(table[:3])
    op.free(otable)
    assert lp.pa_pool_num_free() == 100 and state_equal(lp, op)


def test_random_scripts_match_bit_for_bit(pa):
    rng = random.Random(3411)
    for trial in range(60):
        nb, bs = rng.randint(1, 40), rng.choice([1, 4, 16, 32])
        order = list(range(nb))
        rng.shuffle(order)
        lp, op = pa.Pool(nb, bs, order), OraclePool(nb, bs, order)
        cap = 64
        seqs = {}            # id -> (lib table array, lib len, oracle table, oracle len)
        nid = 0
        for _ in range(250):
            r = rng.random()
            if r < 0.5 and seqs:
                sid = rng.choice(list(seqs))
                t, n, ot, on = seqs[sid]
                try:
                    res = lp.pa_seq_reserve_slot(t, n)
                    lib_err = None
                except pa.PoolExhausted:
                    res, lib_err = None, "exhausted"
                try:
                    ores = op.reserve_slot(ot, on)
                    ora_err = None
                except PoolExhausted:
                    ores, ora_err = None, "exhausted"
                assert lib_err == ora_err
                if res is not None:
                    assert res == ores
                    seqs[sid] = (t, res[1], ot, ores[1])
            elif r < 0.65:
                seqs[nid] = (np.full(cap, -1, np.int32), 0, [], 0)
                nid += 1
            elif r < 0.8 and seqs:
                sid = rng.choice(list(seqs))
                t, n, ot, on = seqs[sid]
                nblk = len(ot)
                lp.pa_pool_fork(t[:nblk])
                op.fork(ot)
                seqs[nid] = (t.copy(), n, list(ot), on)
                nid += 1
            elif seqs:
                sid = rng.choice(list(seqs))
                t, n, ot, on = seqs.pop(sid)
                lp.pa_pool_free(t[: len(ot)])
                op.free(ot)
            for t, n, ot, on in seqs.values():
                assert n == on and list(t[: len(ot)]) == ot
            assert state_equal(lp, op)


def test_batched_reservation_matches_and_rolls_back(pa):
    rng = np.random.default_rng(5)
    nb, bs, cap = 30, 4, 16
    order = rng.permutation(nb)
    lp, op = pa.Pool(nb, bs, order), OraclePool(nb, bs, order)
    lens = np.array([3, 0, 7, 4], np.int32)
    tables = np.full((4, cap), -1, np.int32)
    otables = [[], [], [], []]
    olens = [0, 0, 0, 0]
    # build lengths token by token on both sides
    for s, target in enumerate([3, 0, 7, 4]):
        n = 0
        for _ in range(target):
            _, n, _, _ = lp.pa_seq_reserve_slot(tables[s], n)
            _, olens[s], _, _ = op.reserve_slot(otables[s], olens[s])
    # share sequence 2 into sequence 3's row position: fork
    lp.pa_pool_fork(tables[2][:2])
    op.fork(otables[2])
    tables[3] = tables[2]
    otables[3] = list(otables[2])
    lens[3] = lens[2]
    olens[3] = olens[2]
    for step in range(3):
        slots, pairs = lp.pa_reserve_slots(tables, lens)
        opairs = []
        for s in range(4):
            oslot, olens[s], src, dst = op.reserve_slot(otables[s], olens[s])
            assert slots[s] == oslot
            if src >= 0:
                opairs.append((src, dst))
        assert [tuple(p) for p in pairs] == opairs
        assert list(lens) == olens and state_equal(lp, op)
    # exhaust the pool: the batch fails and nothing changes
    lp.pa_pool_alloc(lp.pa_pool_num_free() - 1)
    op.alloc(op.num_free() - 1)
    before = (tables.copy(), lens.copy(), lp.pa_pool_export())
    grow = np.array([16, 0, 16, 16], np.int32)     # all at block boundaries -> 3 blocks needed, 1 free
    lens[:] = grow
    before = (tables.copy(), lens.copy(), lp.pa_pool_export())
    with pytest.raises(pa.PoolExhausted):
        lp.pa_reserve_slots(tables, lens)
    assert np.array_equal(tables, before[0]) and np.array_equal(lens, before[1])
    after = lp.pa_pool_export()
    assert np.array_equal(after[0], before[2][0]) and np.array_equal(after[1], before[2][1])


def test_errors_match(pa):
    lp, op = pa.Pool(4, 4), OraclePool(4, 4)
    ids = lp.pa_pool_alloc(2)
    assert list(ids) == op.alloc(2)
    with pytest.raises(pa.PagedAttnError) as e:
        lp.pa_pool_free([ids[0], ids[0]])
    assert e.value.status == pa.PA_ERR_REFCOUNT
    with pytest.raises(RefcountError):
        op.free([ids[0], ids[0]])
    with pytest.raises(pa.PagedAttnError) as e:
        lp.pa_pool_fork([3])
    assert e.value.status == pa.PA_ERR_REFCOUNT
    with pytest.raises(pa.PagedAttnError) as e:
        lp.pa_pool_free([17])
    assert e.value.status == pa.PA_ERR_INVALID
    with pytest.raises(InvalidRequest):
        op.free([17])
    with pytest.raises(pa.PoolExhausted):
        lp.pa_pool_alloc(3)
    assert "exhausted" in pa.pa_last_error()
    assert state_equal(lp, op)
    with pytest.raises(pa.PagedAttnError):
        pa.Pool(3, 16, [0, 0, 1])


def test_workload_tables_match_at_full_size(pa):
    """Tables of the Llama-3-8B-shaped workload: library and oracle agree."""
    w = workloads.get("llama3_8b_gqa")
    lens = workloads.lengths(w)
    order = workloads.pool_order(w.num_blocks, w.seed)
    lp, op = pa.Pool(w.num_blocks, w.block_size, order), OraclePool(w.num_blocks, w.block_size, order)
    for n in lens:
        need = -(-int(n) // w.block_size)
        assert list(lp.pa_pool_alloc(need)) == op.alloc(need)
    assert state_equal(lp, op)


def test_reservation_lists_exactly_the_entries_it_wrote(pa):
    """pa_reserve_slots_with_updates: slots and pairs as the oracle's reservations, and the
    (row, column, id) list equal to a diff of the host tables before and after the step."""
    rng = np.random.default_rng(17)
    for trial in range(20):
        bs = int(rng.choice([1, 4, 16]))
        s = int(rng.integers(1, 12))
        cap = 24
        nb = s * cap + 8
        order = rng.permutation(nb)
        lp, op = pa.Pool(nb, bs, order), OraclePool(nb, bs, order)
        tables = np.full((s, cap), -1, np.int32)
        lens = np.zeros(s, np.int32)
        otables, olens = [[] for _ in range(s)], [0] * s
        for r in range(s):
            target = int(rng.integers(0, cap * bs // 2))
            for _ in range(target):
                _, lens[r], _, _ = lp.pa_seq_reserve_slot(tables[r], lens[r])
                _, olens[r], _, _ = op.reserve_slot(otables[r], olens[r])
        # some rows become forks of their neighbour (shared blocks -> copy-on-write)
        for r in range(1, s):
            if rng.random() < 0.4 and lens[r - 1] > 0:
                n = -(-int(lens[r - 1]) // bs)
                lp.pa_pool_free(tables[r, :-(-int(lens[r]) // bs)]) if lens[r] else None
                op.free(otables[r]) if otables[r] else None
                lp.pa_pool_fork(tables[r - 1, :n])
                op.fork(otables[r - 1])
                tables[r] = tables[r - 1]
                lens[r] = lens[r - 1]
                otables[r], olens[r] = list(otables[r - 1]), olens[r - 1]
        row0 = int(rng.integers(0, 5))
        for step in range(int(rng.integers(1, 2 * bs + 2))):
            before = tables.copy()
            slots = np.empty(s, np.int64)
            pairs = np.empty((s, 2), np.int32)
            upd = np.full((s, 3), -7, np.int32)
            npairs, nupd = lp.pa_reserve_slots_with_updates(tables, lens, row0, slots, pairs, upd)
            opairs = []
            for r in range(s):
                oslot, olens[r], src, dst = op.reserve_slot(otables[r], olens[r])
                assert slots[r] == oslot
                if src >= 0:
                    opairs.append((src, dst))
            assert [tuple(p) for p in pairs[:npairs]] == opairs
            rows, cols = np.nonzero(tables != before)
            expect = sorted((int(r) + row0, int(c), int(tables[r, c])) for r, c in zip(rows, cols))
            assert sorted(tuple(int(x) for x in u) for u in upd[:nupd]) == expect
            assert list(lens) == olens and state_equal(lp, op)
