"""Decode calls queued back to back on one stream, sharing one workspace.

Each call's planner resets the work counter and rewrites the work list at
the head of the workspace, while the decode grid of the call before it on the
stream may still be taking units from that list: the planner therefore waits
for the kernel before it to finish before it touches the workspace (or reads
the lengths).  These tests queue several calls with different queries,
lengths and outputs on one stream and one workspace, with no synchronisation
between them, and compare every call's output with the oracle.

The calls share one cache and one set of block tables in which every entry
names a valid, filled block, and the same batch size and table width, so a
call that ran another call's work units would give wrong numbers, never an
out-of-range access.  Attention is the single-query decode over the block
table ("PagedAttention Explained: Managing KV Cache Efficiently", section
"Block Tables and Non-Contiguous Storage").
"""

import math

import numpy as np
import pytest
import torch

from oracle import oracle_decode
from gpu_cases import AsF64, assert_close, full_table_case
from paged_kv_cache_341_b200 import workloads

pytestmark = pytest.mark.gpu

S, MB, BS, HQ, HKV, D = 64, 64, 16, 32, 8, 128


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa as mod
    assert mod.pa_device_error(reset=True) == 0
    return mod


@pytest.fixture(scope="module")
def case(pa):
    cache, k, v, tables = full_table_case(S, MB, BS, HKV, D, "bf16", seed=4101)
    rng = np.random.default_rng(4102)
    cap = MB * BS
    lens_sets = [
        [int(x) for x in rng.integers(cap // 2, cap + 1, size=S)],     # long
        [int(x) for x in rng.integers(1, 200, size=S)],                # short
        [int(x) for x in rng.integers(0, cap + 1, size=S)],            # mixed, with empty rows
        [cap] * (S // 2) + [1] * (S - S // 2),                         # full rows then single tokens
    ]
    qs = [workloads.randn((S, HQ, D), "bf16", 4110 + i) for i in range(4)]
    return cache, AsF64(k), AsF64(v), tables, lens_sets, qs


def queue_calls(pa, case, partition):
    """Issue four calls back to back on the current stream, then synchronise once."""
    cache, _, _, _, lens_sets, qs = case
    scale = 1.0 / math.sqrt(D)
    d_lens = [torch.tensor(l, dtype=torch.int32, device="cuda") for l in lens_sets]
    d_q = [q.cuda() for q in qs]
    outs = [torch.full((S, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    ws = pa.decode_workspace(S, HQ, D, MB, BS, partition)
    assert ws is not None                           # even a single pass plans through the workspace
    torch.cuda.synchronize()
    for i in range(4):
        pa.pa_decode_attention(d_q[i], cache.k_cache, cache.v_cache, cache.d_tables, d_lens[i], scale, outs[i],
                               partition_size=partition, workspace=ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    return [o.float().cpu().numpy() for o in outs]


def check_against_oracle(case, outs, where):
    _, kd, vd, tables, lens_sets, qs = case
    scale = 1.0 / math.sqrt(D)
    for i, got in enumerate(outs):
        ref = oracle_decode(qs[i].double().numpy(), kd, vd, tables, lens_sets[i], scale)
        assert_close(got, ref, "bf16", "%s, call %d" % (where, i))


@pytest.mark.parametrize("partition", [0, 512, 256])
def test_back_to_back_calls_share_a_workspace(pa, case, partition):
    outs = queue_calls(pa, case, partition)
    check_against_oracle(case, outs, "partition %d" % partition)
