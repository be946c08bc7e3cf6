"""The native step executor (pa_engine_*) against the oracle: many decode steps
from host buffers, with fresh blocks at block boundaries, a copy-on-write of a
shared block, steps over a sub-range of the batch, and pool exhaustion.

Per step the oracle takes the same path the pages describe: reserve the slot
(fresh block at offset 0, private copy of a shared partly filled block), copy,
append the new token's K/V, then attend over the gathered blocks."""

import math

import numpy as np
import pytest
import torch

from gpu_cases import TORCH, AsF64, assert_close
from oracle import OraclePool, oracle_append, oracle_copy_blocks, oracle_decode
from paged_kv_cache_341_b200 import workloads

pytestmark = pytest.mark.gpu


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa
    from paged_kv_cache_341_b200.cache import PagedKVCache
    return pa, PagedKVCache


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def _setup(PagedKVCache, dtype, nb, bs, hkv, d, lens0, share, max_blocks, seed):
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    rows = len(lens0) + len(share)
    cache = PagedKVCache(nb, bs, hkv, d, TORCH[dtype], rows, max_blocks, initial_free_order=order,
                         fill=float("nan"))
    opool = OraclePool(nb, bs, order)
    otables, olens = [[] for _ in range(rows)], [0] * rows
    for r, n in enumerate(lens0):
        cache.allocate(r, n)
        otables[r] = opool.alloc(-(-n // bs))
        olens[r] = n
    for dst, src in share:
        cache.share(src, dst)
        opool.fork(otables[src])
        otables[dst], olens[dst] = list(otables[src]), olens[src]
    k_host = torch.full(cache.k_cache.shape, float("nan"), dtype=TORCH[dtype])
    v_host = torch.full_like(k_host, float("nan"))
    ids = sorted({b for t in otables for b in t})
    k_host[ids] = workloads.randn((len(ids), bs, hkv, d), dtype, seed + 1)
    v_host[ids] = workloads.randn((len(ids), bs, hkv, d), dtype, seed + 2)
    cache.k_cache.copy_(k_host)
    cache.v_cache.copy_(v_host)
    return cache, opool, otables, olens, k_host, v_host


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("part", [0, 16, 32])
def test_engine_steps_match_oracle(dtype, part):
    pa, PagedKVCache = _lib()
    nb, bs, hq, hkv, d = 64, 16, 8, 2, 128
    lens0 = [1, 15, 16, 17, 40]
    cache, opool, otables, olens, k_host, v_host = _setup(PagedKVCache, dtype, nb, bs, hkv, d, lens0, [(5, 4)],
                                                          8, 3400 + part)
    rows = len(otables)
    scale = 1 / math.sqrt(d)
    eng = cache.engine(hq, part)
    steps = []
    n_pairs = 0
    for i in range(20):
        row0, n = (2, 3) if i % 3 == 2 else (0, rows)
        seed = 9000 + 10 * i
        q = workloads.randn((n, hq, d), dtype, seed).pin_memory()
        kn = workloads.randn((n, hkv, d), dtype, seed + 1).pin_memory()
        vn = workloads.randn((n, hkv, d), dtype, seed + 2).pin_memory()
        out = torch.empty((n, hq, d), dtype=TORCH[dtype]).pin_memory()
        slots, pairs = eng.pa_engine_step(row0, n, q, kn, vn, out, scale, want_slots=True)
        # the oracle's step for the same rows
        oslots, opairs = [], []
        for r in range(row0, row0 + n):
            slot, olens[r], src, dst = opool.reserve_slot(otables[r], olens[r])
            oslots.append(slot)
            if src >= 0:
                opairs.append((src, dst))
        assert list(slots) == oslots, "step %d slots" % i
        assert [tuple(p) for p in pairs] == opairs, "step %d pairs" % i
        n_pairs += len(opairs)
        oracle_copy_blocks(k_host, v_host, opairs)
        oracle_append(k_host, v_host, kn, vn, oslots)
        ref = oracle_decode(q.double().numpy(), AsF64(k_host), AsF64(v_host), otables[row0:row0 + n],
                            olens[row0:row0 + n], scale)
        steps.append((q, kn, vn, out, ref, row0, n))
    eng.pa_engine_synchronize()
    assert pa.pa_device_error() == 0
    for i, (_, _, _, out, ref, row0, n) in enumerate(steps):
        assert_close(out.double().numpy(), ref, dtype, "step %d rows %d..%d" % (i, row0, row0 + n))
    # exactly one copy-on-write happened (row 4 writing into the block it shares with row 5)
    assert n_pairs == 1
    assert torch.equal(_bits(cache.k_cache.cpu()), _bits(k_host))
    assert torch.equal(_bits(cache.v_cache.cpu()), _bits(v_host))
    for r in range(rows):
        nblk = -(-olens[r] // bs)
        assert list(cache.tables[r, :nblk]) == otables[r]
        assert list(cache.d_tables[r, :nblk].cpu().numpy()) == otables[r]
    assert list(cache.lens) == olens and list(cache.d_lens.cpu().numpy()) == olens
    refs, free = cache.pool.pa_pool_export()
    orefs, ofree = opool.export()
    assert list(refs) == orefs and list(free) == ofree
    eng.close()


def test_engine_copy_on_write_pair_reported_once():
    pa, PagedKVCache = _lib()
    nb, bs, hq, hkv, d = 16, 16, 4, 1, 64
    cache, opool, otables, olens, k_host, v_host = _setup(PagedKVCache, "bf16", nb, bs, hkv, d, [20], [(1, 0)], 4,
                                                          77)
    eng = cache.engine(hq, 0)
    q = workloads.randn((2, hq, d), "bf16", 1).pin_memory()
    kn = workloads.randn((2, hkv, d), "bf16", 2).pin_memory()
    vn = workloads.randn((2, hkv, d), "bf16", 3).pin_memory()
    out = torch.empty((2, hq, d), dtype=torch.bfloat16).pin_memory()
    slots, pairs = eng.pa_engine_step(0, 2, q, kn, vn, out, 0.125, want_slots=True)
    eng.pa_engine_synchronize()
    # row 0 moves onto a private copy of its last block; row 1 then owns the original alone
    assert pairs.shape == (1, 2) and pairs[0, 0] == otables[0][1]
    assert cache.pool.pa_pool_refcount(int(pairs[0, 0])) == 1 and cache.pool.pa_pool_refcount(int(pairs[0, 1])) == 1
    assert torch.equal(_bits(cache.k_cache[int(pairs[0, 1]), :4].cpu()), _bits(k_host[int(pairs[0, 0]), :4]))
    eng.close()


def test_engine_exhaustion_leaves_everything_unchanged():
    pa, PagedKVCache = _lib()
    nb, bs, hq, hkv, d = 4, 16, 4, 2, 64
    cache, opool, otables, olens, k_host, v_host = _setup(PagedKVCache, "bf16", nb, bs, hkv, d, [16, 16], [], 4, 5)
    eng = cache.engine(hq, 0)
    bufs = []

    def step():
        q = workloads.randn((2, hq, d), "bf16", len(bufs)).pin_memory()
        kn = workloads.randn((2, hkv, d), "bf16", 50 + len(bufs)).pin_memory()
        out = torch.empty((2, hq, d), dtype=torch.bfloat16).pin_memory()
        bufs.append((q, kn, out))
        return eng.pa_engine_step(0, 2, q, kn, kn, out, 0.125)

    for _ in range(16):         # rows grow 16 -> 32 (both take their second block: the pool is now empty)
        step()
    eng.pa_engine_synchronize()
    tables, lens = cache.tables.copy(), cache.lens.copy()
    refs, free = cache.pool.pa_pool_export()
    with pytest.raises(pa.PoolExhausted):
        step()
    assert np.array_equal(cache.tables, tables) and np.array_equal(cache.lens, lens)
    refs2, free2 = cache.pool.pa_pool_export()
    assert np.array_equal(refs, refs2) and np.array_equal(free, free2)
    eng.pa_engine_synchronize()
    assert pa.pa_device_error() == 0
    eng.close()


def test_engine_with_pageable_host_buffers():
    pa, PagedKVCache = _lib()
    nb, bs, hq, hkv, d = 32, 16, 8, 2, 128
    cache, opool, otables, olens, k_host, v_host = _setup(PagedKVCache, "bf16", nb, bs, hkv, d, [33, 7, 64], [], 8,
                                                          11)
    eng = cache.engine(hq, 32)
    outs = []
    for i in range(3):
        q = workloads.randn((3, hq, d), "bf16", 60 + i)          # ordinary (pageable) host memory
        kn = workloads.randn((3, hkv, d), "bf16", 70 + i)
        vn = workloads.randn((3, hkv, d), "bf16", 80 + i)
        out = torch.empty((3, hq, d), dtype=torch.bfloat16)
        slots, _ = eng.pa_engine_step(0, 3, q, kn, vn, out, 0.1, want_slots=True)
        oslots = []
        for r in range(3):
            slot, olens[r], _, _ = opool.reserve_slot(otables[r], olens[r])
            oslots.append(slot)
        assert list(slots) == oslots
        oracle_append(k_host, v_host, kn, vn, oslots)
        outs.append((out, oracle_decode(q.double().numpy(), AsF64(k_host), AsF64(v_host), otables, olens, 0.1),
                     q, kn, vn))
    eng.pa_engine_synchronize()
    for i, (out, ref, *_) in enumerate(outs):
        assert_close(out.double().numpy(), ref, "bf16", "pageable step %d" % i)
    eng.close()


def test_engine_rejects_bad_rows_and_buffers():
    pa, PagedKVCache = _lib()
    cache, *_ = _setup(PagedKVCache, "bf16", 8, 16, 2, 64, [5, 9], [], 2, 1)
    eng = cache.engine(4, 0)
    q = torch.zeros((2, 4, 64), dtype=torch.bfloat16)
    kn = torch.zeros((2, 2, 64), dtype=torch.bfloat16)
    out = torch.empty_like(q)
    lib = pa._lib
    fake = q.data_ptr()
    import ctypes
    vp = ctypes.c_void_p
    assert lib.pa_engine_step(eng._h, 1, 2, vp(fake), vp(fake), vp(fake), vp(fake), 1.0, None, None,
                              None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_step(eng._h, -1, 1, vp(fake), vp(fake), vp(fake), vp(fake), 1.0, None, None,
                              None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_step(eng._h, 0, 2, vp(fake), vp(fake), vp(fake), vp(fake), float("nan"), None, None,
                              None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_step(eng._h, 0, 2, None, vp(fake), vp(fake), vp(fake), 1.0, None, None,
                              None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_step(eng._h, 0, 0, None, None, None, None, 1.0, None, None, None) == pa.PA_OK
    with pytest.raises(TypeError):
        eng.pa_engine_step(0, 2, q.cuda(), kn, kn, out, 1.0)
    assert list(cache.lens) == [5, 9]          # nothing was reserved
    eng.close()
