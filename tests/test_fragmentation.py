"""Fragmentation simulator (host only): the contiguous arena and the replay
loop against closed forms, and the library pool against the oracle pool on
the same trace."""

import numpy as np
import pytest

from oracle import OraclePool
from paged_kv_cache_341_b200 import build

build.ensure_built()
from paged_kv_cache_341_b200 import fragmentation as fr  # noqa: E402
from paged_kv_cache_341_b200 import pa  # noqa: E402


def test_arena_external_fragmentation_example():
    # three buffers of 3 in 10 slots; the middle one leaves: 4 slots free in
    # two holes (3 + 1), yet 4 contiguous slots cannot be had
    a = fr.ContiguousArena(10)
    assert [a.alloc(3), a.alloc(3), a.alloc(3)] == [0, 3, 6]
    a.free(3, 3)
    assert a.free_total() == 4 and a.largest_hole() == 3
    assert a.alloc(4) is None
    a.free(0, 3)                       # neighbours merge into one hole of 6
    assert a.holes == [(0, 6), (9, 1)]
    assert a.alloc(4) == 0
    a.free(0, 4)
    a.free(6, 3)
    assert a.holes == [(0, 10)]


def test_static_waste_of_the_pages_example():
    # a 2,048-token reservation that ends up holding 200 tokens
    assert fr.static_waste([200], 2048) == pytest.approx(1 - 200 / 2048)
    assert fr.static_waste([2048, 1024], 2048) == pytest.approx(0.25)


@pytest.mark.parametrize("p,o", [(5, 30), (16, 16), (1, 1), (100, 250)])
def test_single_request_closed_forms(p, o):
    trace = [fr.Request(0, p, o)]
    m = 1024
    # contiguous, maximum context: after step t the request holds p + t of m slots, t = 1..o
    r = fr.simulate(trace, 4096, "contiguous-max", max_context=m)
    used = sum(p + t for t in range(1, o + 1))
    assert (r.steps, r.finished, r.used_slot_steps, r.held_slot_steps) == (o, 1, used, o * m)
    assert r.waste == pytest.approx(1 - used / (o * m))
    # exact reservation holds p + o slots throughout
    r = fr.simulate(trace, 4096, "contiguous-exact", max_context=m)
    assert r.held_slot_steps == o * (p + o) and r.used_slot_steps == used
    # paged: ceil(L / bs) blocks of bs slots at length L
    for bs in (8, 16, 32):
        r = fr.simulate(trace, 4096, "paged", block_size=bs, max_context=m)
        held = sum(-(-(p + t) // bs) * bs for t in range(1, o + 1))
        assert r.held_slot_steps == held and r.used_slot_steps == used and r.preemptions == 0


def test_paged_slack_is_below_one_block_per_sequence():
    trace = fr.synthetic_trace(150, 2048, seed=7, rate=6.0)
    for bs in (8, 16, 32):
        r = fr.simulate(trace, 48 * 1024, "paged", block_size=bs)
        assert r.finished == len(trace) and r.external_failures == 0
        assert 0 <= r.held_slot_steps - r.used_slot_steps <= (bs - 1) * r.running_steps


def test_everything_is_returned_to_the_pool():
    pools = []

    def factory(nb, bs):
        pools.append(pa.Pool(nb, bs))
        return pools[-1]

    trace = fr.synthetic_trace(120, 2048, seed=11, rate=8.0)
    r = fr.simulate(trace, 16 * 1024, "paged", pool_factory=factory)
    assert r.finished == len(trace) and r.preemptions > 0     # the budget is tight enough to preempt
    assert pools[0].pa_pool_num_free() == 16 * 1024 // 16
    refs, _ = pools[0].pa_pool_export()
    assert not refs.any()


def test_library_pool_replays_like_the_oracle_pool():
    trace = fr.synthetic_trace(60, 1024, seed=5, rate=8.0, prompt=(16, 256), output_median=96)
    for bs in (8, 16):
        lib = fr.simulate(trace, 6 * 1024, "paged", block_size=bs, max_context=1024)
        ora = fr.simulate(trace, 6 * 1024, "paged", block_size=bs, max_context=1024,
                          pool_factory=lambda nb, b: OraclePool(nb, b))
        assert lib == ora
        assert lib.preemptions > 0


def test_paged_holds_less_than_contiguous_on_the_synthetic_trace():
    trace = fr.synthetic_trace(200, 2048, seed=3414)
    cmax = fr.simulate(trace, 32 * 2048, "contiguous-max")
    cex = fr.simulate(trace, 32 * 2048, "contiguous-exact")
    paged = fr.simulate(trace, 32 * 2048, "paged")
    # the pages' range for reservations sized to the maximum context
    assert 0.6 <= cmax.waste <= 0.8
    assert paged.waste < 0.02 < cex.waste < cmax.waste
    assert paged.mean_batch > cex.mean_batch > cmax.mean_batch
    assert paged.steps < cmax.steps
