"""Full-size workloads on the GPU, in the launch configuration the benchmark
times: one decode step (reserve, copy-on-write, append, partitioned
attention with the workload's partition size plus the merge), checked
against the oracle replaying the same steps.

* block tables, slots, copy pairs and pool state: bit-exact;
* appended rows and copied blocks: bit-exact;
* attention: every (sequence, query head) output against the oracle for the
  Llama-2-7B, Llama-3-8B and 70B-shaped workloads; for the shared-prefix
  workload (200 sequences x 30,720 + suffix tokens, about 100 GFLOP of
  float64 work for all of them) a stratified sample of sequences covering
  every 128-row query tile of the prefix kernel, all heads, against the
  oracle, and every output of the cascade call against the plain call.

The shared-prefix workload is the "Paged Attention" glossary's example (a
30k-token prompt shared by 200 users; aidolsgroup.com, section "Example") and
agentechip.com's "Shared Prefix Caching".
"""

import math

import numpy as np
import pytest
import torch

from oracle import OraclePool, oracle_append, oracle_copy_blocks, oracle_decode
from gpu_cases import AsF64, assert_close
from paged_kv_cache_341_b200 import workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def oracle_replay(sc):
    """Allocate the workload's tables with the oracle pool, independently of the library."""
    w = sc.w
    op = OraclePool(w.num_blocks, w.block_size, workloads.pool_order(w.num_blocks, w.seed))
    s = w.num_seqs
    if w.shared_prefix:
        prefix = op.alloc(w.shared_prefix // w.block_size)
        tables = [list(prefix)]
        for _ in range(1, s):
            op.fork(prefix)
            tables.append(list(prefix))
        lens = []
        for r in range(s):
            tables[r] = tables[r] + op.alloc(-(-int(sc.lens0[r]) // w.block_size))
            lens.append(w.shared_prefix + int(sc.lens0[r]))
        for r in range(s):
            op.fork(tables[r])
            tables.append(list(tables[r]))
            lens.append(lens[r])
    else:
        tables, lens = [], []
        for n in sc.lens0:
            tables.append(op.alloc(-(-int(n) // w.block_size)))
            lens.append(int(n))
    return op, tables, lens


def prefix_tile_sample(batch, group, rng, per_tile=4):
    """Sequences covering every 128-row query tile of one KV head (rows s * group + g):
    the first and last sequence of each tile and ``per_tile - 2`` others."""
    seqs_per_tile = 128 // group
    picks = set()
    for t0 in range(0, batch, seqs_per_tile):
        t1 = min(batch, t0 + seqs_per_tile) - 1
        picks |= {t0, t1}
        inner = list(range(t0 + 1, t1))
        if inner:
            picks |= set(int(x) for x in rng.choice(inner, min(per_tile - 2, len(inner)), replace=False))
    return sorted(picks)


def full_step(name):
    """Build the workload, take one decode step through the library and the oracle; check the
    bit-exact parts.  Returns what the attention checks need."""
    from paged_kv_cache_341_b200 import pa
    from paged_kv_cache_341_b200.scenarios import Scenario
    sc = Scenario(name, keep_host=True)
    w, c = sc.w, sc.cache
    op, otables, olens = oracle_replay(sc)
    for r in range(c.num_seqs):
        nblk = -(-olens[r] // w.block_size)
        assert int(c.lens[r]) == olens[r] and list(c.tables[r, :nblk]) == otables[r]
    refs, free = c.pool.pa_pool_export()
    orefs, ofree = op.export()
    assert list(refs) == orefs and list(free) == ofree
    if w.shared_prefix:
        assert orefs[otables[0][0]] == 2 * w.num_seqs       # prefix block: 200 sequences + 200 forks

    # one decode step through the library
    q, k_new, v_new = sc.step_inputs(0)
    out = torch.full((sc.batch, w.num_q_heads, w.head_dim), float("nan"), dtype=w.torch_dtype, device="cuda")
    ws = pa.decode_workspace(sc.batch, w.num_q_heads, w.head_dim, c.max_blocks, w.block_size, w.partition_size)
    q_dev = q.cuda()
    slots, pairs = c.decode_step(q_dev, k_new.cuda(), v_new.cuda(), out, w.scale, w.partition_size, ws,
                                 rows=sc.rows)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0

    # the oracle takes the same step on the host copy
    oslots, opairs = [], []
    for r in range(sc.rows.start, sc.rows.stop):
        slot, olens[r], src, dst = op.reserve_slot(otables[r], olens[r])
        oslots.append(slot)
        if src >= 0:
            opairs.append((src, dst))
    assert list(slots) == oslots and [tuple(p) for p in pairs] == opairs
    if w.shared_prefix:
        expect_cow = sum(1 for n in sc.lens0 if int(n) % w.block_size)
        assert len(opairs) == expect_cow > 0
    oracle_copy_blocks(sc.k_host, sc.v_host, opairs)
    oracle_append(sc.k_host, sc.v_host, k_new, v_new, oslots)

    # the device tables followed the host reservation (entries applied incrementally)
    for r in range(sc.rows.start, sc.rows.stop):
        nblk = -(-olens[r] // w.block_size)
        assert list(c.d_tables[r, :nblk].cpu().numpy()) == otables[r]
    assert list(c.d_lens.cpu().numpy()) == olens

    # bit-exact: appended rows and every copied block
    flat_k = c.k_cache.view(-1, w.num_kv_heads, w.head_dim)
    flat_v = c.v_cache.view(-1, w.num_kv_heads, w.head_dim)
    idx = torch.tensor(oslots, dtype=torch.int64, device="cuda")
    assert torch.equal(flat_k[idx].cpu(), k_new) and torch.equal(flat_v[idx].cpu(), v_new)
    for src, dst in opairs:
        assert torch.equal(c.k_cache[dst].cpu(), sc.k_host[dst]) and torch.equal(c.v_cache[dst].cpu(), sc.v_host[dst])

    btables = otables[sc.rows.start:sc.rows.stop]
    blens = [int(x) for x in olens[sc.rows.start:sc.rows.stop]]
    return sc, q, q_dev, out, btables, blens


@pytest.mark.parametrize("name", ["llama2_7b_mha", "llama3_8b_gqa", "long_70b_gqa"])
def test_full_size_step(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sc, q, _, out, btables, blens = full_step(name)
    w = sc.w
    ref = oracle_decode(q.double().numpy(), AsF64(sc.k_host), AsF64(sc.v_host), btables, blens, w.scale)
    assert_close(out.float().cpu().numpy(), ref, w.dtype, "%s, every (sequence, head)" % name)


@pytest.mark.parametrize("prefix_path", ["pair", "umma"])
def test_shared_prefix_full_size_step_plain_and_cascade(monkeypatch, prefix_path):
    """The shared-prefix step: copy-on-write of the forks' partly filled last blocks, append,
    then attention twice over the same state -- the plain partitioned call and the cascade
    call (prefix once for all 200 x 32 query rows on a tcgen05 kernel -- the SM-pair one, the
    default, or the one-SM one -- 60 slices of 512 tokens, suffix partitions of 512, merge)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import pa
    sc, q, q_dev, plain, btables, blens = full_step("shared_prefix")
    w, c = sc.w, sc.cache
    monkeypatch.setenv("PA_PREFIX_PATH", prefix_path)
    pblocks = w.shared_prefix // w.block_size
    prefix_ids = c.d_tables[sc.rows.start, :pblocks].contiguous()
    suffix_tables = c.d_tables[sc.rows, pblocks:]
    suffix_lens = (c.d_lens[sc.rows] - w.shared_prefix).contiguous()
    ws = torch.empty(pa.pa_shared_prefix_workspace_size(sc.batch, w.num_q_heads, w.head_dim, w.shared_prefix,
                                                        suffix_tables.shape[1], w.block_size, w.partition_size),
                     dtype=torch.uint8, device="cuda")
    casc = torch.full_like(plain, float("nan"))
    pa.pa_decode_attention_shared_prefix(q_dev, c.k_cache, c.v_cache, prefix_ids, w.shared_prefix, suffix_tables,
                                         suffix_lens, w.scale, casc, w.partition_size, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    assert pa.pa_debug_last_prefix_kernel() == {"pair": 1, "umma": 2}[prefix_path]
    for r in range(sc.batch):
        assert btables[r][:pblocks] == btables[0][:pblocks]
    plain_h = plain.float().cpu().numpy()
    casc_h = casc.float().cpu().numpy()
    assert_close(casc_h, plain_h, w.dtype, "cascade vs plain call, all 200 x 32 outputs")
    group = w.num_q_heads // w.num_kv_heads
    picks = prefix_tile_sample(sc.batch, group, np.random.default_rng(341))
    assert len(picks) >= 24 and picks[-1] == sc.batch - 1
    ref = oracle_decode(q.double().numpy(), AsF64(sc.k_host), AsF64(sc.v_host), btables, blens, w.scale, seqs=picks)
    assert_close(plain_h[picks], ref[picks], w.dtype, "plain call, %d sampled sequences" % len(picks))
    assert_close(casc_h[picks], ref[picks], w.dtype, "cascade call, %d sampled sequences" % len(picks))
