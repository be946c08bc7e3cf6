"""Full-size workloads on the GPU, in the launch configuration the benchmark
times (one decode step: reserve, copy-on-write, append, partitioned attention
with 512-token partitions), checked against the oracle replaying the same
steps: block tables, slots, copy pairs and pool state bit-exact, appended
rows and copied blocks bit-exact, and attention on sampled (sequence, head)
outputs within tolerance (every output must be finite)."""

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


@pytest.mark.parametrize("name", ["llama2_7b_mha", "llama3_8b_gqa", "shared_prefix", "long_70b_gqa"])
def test_full_size_step(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
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
    slots, pairs = c.decode_step(q.cuda(), k_new.cuda(), v_new.cuda(), out, w.scale, w.partition_size, ws,
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

    # bit-exact: appended rows and copied blocks
    flat_k = c.k_cache.view(-1, w.num_kv_heads, w.head_dim)
    flat_v = c.v_cache.view(-1, w.num_kv_heads, w.head_dim)
    idx = torch.tensor(oslots, dtype=torch.int64, device="cuda")
    assert torch.equal(flat_k[idx].cpu(), k_new) and torch.equal(flat_v[idx].cpu(), v_new)
    for src, dst in opairs[:64]:
        assert torch.equal(c.k_cache[dst].cpu(), sc.k_host[dst]) and torch.equal(c.v_cache[dst].cpu(), sc.v_host[dst])

    # attention: every output finite; sampled outputs against the oracle
    gpu = out.float().cpu().numpy()
    assert np.all(np.isfinite(gpu))
    rng = np.random.default_rng(341)
    blens = np.array(olens[sc.rows.start:sc.rows.stop])
    picks = {int(np.argmax(blens)), int(np.argmin(blens))} | set(int(x) for x in rng.choice(sc.batch, min(10, sc.batch), False))
    btables = otables[sc.rows.start:sc.rows.stop]
    kw, vw = AsF64(sc.k_host), AsF64(sc.v_host)
    qd = q.double().numpy()
    for sidx in sorted(picks):
        heads = sorted(set(int(h) for h in rng.choice(w.num_q_heads, 4, False)) | {0, w.num_q_heads - 1})
        ref = oracle_decode(qd, kw, vw, btables, blens, w.scale, seqs=[sidx], heads=heads)
        assert_close(gpu[sidx, heads], ref[sidx, heads], w.dtype, "%s seq %d" % (name, sidx))
