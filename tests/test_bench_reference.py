"""The reference arm of bench.py times the oracle on the step the GPU arm times: one slot reserved per
sequence (copy-on-write of a shared partly filled block), the step's new K/V written there, and
attention over len + 1 tokens. Host only."""

import numpy as np
import pytest

import bench
from oracle import OraclePool
from paged_kv_cache_341_b200 import workloads


@pytest.mark.parametrize("name", ["tiny_fp32"])
def test_reference_scenario_is_the_timed_step(name):
    sc = bench.ReferenceScenario(name)
    w = sc.w
    lens0 = workloads.lengths(w) + w.shared_prefix
    rows = range(sc.rows.start, sc.rows.stop)
    assert [int(sc.cache.lens[r]) for r in rows] == [int(n) + 1 for n in lens0]
    # the new token of each sequence sits where the FIFO pool puts token number len, with the step's K/V
    _, k_new, v_new = sc.step_inputs(0)
    op = OraclePool(w.num_blocks, w.block_size, workloads.pool_order(w.num_blocks, w.seed))
    tables = []
    for n in lens0:
        ids = op.alloc(-(-int(n) // w.block_size))
        tables.append(list(ids))
    for i, (r, n) in enumerate(zip(rows, lens0)):
        slot, n1, src, dst = op.reserve_slot(tables[i], int(n))
        assert n1 == int(n) + 1 and src == -1
        assert list(sc.cache.tables[r, :len(tables[i])]) == tables[i]
        blk, off = divmod(slot, w.block_size)
        assert np.array_equal(sc.k_host[blk, off].numpy(), k_new[i].numpy())
        assert np.array_equal(sc.v_host[blk, off].numpy(), v_new[i].numpy())


def test_reference_config_matches_the_reserved_lengths():
    sc = bench.ReferenceScenario("tiny_fp32")

    class A:
        gpus = 1
        partition = None
    cfg = bench.workload_config(sc, A())
    lens = sc.cache.lens[sc.rows]
    assert cfg["mean_context"] == round(float(np.mean(lens)), 1)
    assert cfg["max_context"] == int(np.max(lens))


def test_call_label_names_the_kernels_that_run(monkeypatch):
    # the roofline's kernel label follows the launch rules: the one-warp
    # planner for batches of up to 32 sequences, the SM-pair prefix kernel
    # unless PA_PREFIX_PATH picks another
    monkeypatch.delenv("PA_PREFIX_PATH", raising=False)
    monkeypatch.delenv("PA_DECODE_PATH", raising=False)
    w70 = workloads.WORKLOADS["long_70b_gqa"]
    w3 = workloads.WORKLOADS["llama3_8b_gqa"]
    wsp = workloads.WORKLOADS["shared_prefix"]
    assert "plan_small_kernel + decode_mma_kernel" in bench.call_label(False, w70, 8, 300, "measured")
    assert "(plan_kernel + decode_mma_kernel" in bench.call_label(False, w3, 256, 300, "measured")
    assert "prefix_pair_kernel + plan_kernel" in bench.call_label(True, wsp, 200, 300, "measured")
    monkeypatch.setenv("PA_PREFIX_PATH", "umma")
    assert "prefix_umma_kernel" in bench.call_label(True, wsp, 200, 300, "measured")
    monkeypatch.setenv("PA_PREFIX_PATH", "mma")
    assert "prefix_attention_kernel" in bench.call_label(True, wsp, 200, 300, "measured")
