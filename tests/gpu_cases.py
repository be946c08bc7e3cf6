"""Shared helpers of the GPU parity tests: build a paged cache through the
library, the same inputs for the oracle, and the tolerance check."""

import numpy as np
import torch

from paged_kv_cache_341_b200 import workloads

TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


class AsF64:
    """View of a CPU torch pool ``[NB, bs, Hkv, D]`` that hands the oracle float64 blocks (exact widening)."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, b):
        return self.t[b].to(torch.float64).numpy()


def assert_close(gpu, ref, dtype, where=""):
    """fp32 cache: max-abs 1e-5.  fp16/bf16: |gpu - ref| <= 2e-2 + 1e-2 |ref| elementwise."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(gpu)), "non-finite output " + where
    err = np.abs(gpu - ref)
    if dtype == "f32":
        bound = np.full_like(ref, 1e-5)
    else:
        bound = 2e-2 + 1e-2 * np.abs(ref)
    bad = err > bound
    assert not bad.any(), "%s: %d of %d outside tolerance, worst %.3g (ref %.3g)" % (
        where, int(bad.sum()), bad.size, float(err.max()), float(ref.flat[int(np.argmax(err))]))
    return float(err.max())


def build_pool_contents(pool_shape, dtype, tables, lens, block_size, seed, poison=True):
    """Host pools with N(0,1) values in every used block and NaN everywhere else
    (including the unused rows of each sequence's last block)."""
    k = torch.full(pool_shape, float("nan") if poison else 0.0, dtype=TORCH[dtype])
    v = torch.full(pool_shape, float("nan") if poison else 0.0, dtype=TORCH[dtype])
    used = []
    for t, n in zip(tables, lens):
        used.extend(int(b) for b in t[: -(-int(n) // block_size)])
    used = sorted(set(used))
    if used:
        ids = torch.tensor(used, dtype=torch.int64)
        sub = (len(used),) + tuple(pool_shape[1:])
        k[ids] = workloads.randn(sub, dtype, seed)
        v[ids] = workloads.randn(sub, dtype, seed + 1)
    if poison:
        for t, n in zip(tables, lens):
            n = int(n)
            if n % block_size:
                last = int(t[n // block_size])
                k[last, n % block_size:] = float("nan")
                v[last, n % block_size:] = float("nan")
    return k, v


def full_table_case(num_seqs, max_blocks, block_size, num_kv_heads, head_dim, dtype, seed):
    """A cache whose every block-table entry names a valid, filled block.

    Each of ``num_seqs`` rows owns ``max_blocks`` blocks (from a seeded
    shuffled pool), so any length up to ``max_blocks * block_size`` can be
    attended without touching an unfilled slot.  Returns (cache, k_host,
    v_host, host tables as lists)."""
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(seed)
    cap = max_blocks * block_size
    nb = num_seqs * max_blocks + 2
    cache = PagedKVCache(nb, block_size, num_kv_heads, head_dim, TORCH[dtype], num_seqs, max_blocks,
                         initial_free_order=rng.permutation(nb))
    for row in range(num_seqs):
        cache.allocate(row, cap)
    full = [cap] * num_seqs
    k, v = build_pool_contents((nb, block_size, num_kv_heads, head_dim), dtype, cache.tables, full, block_size,
                               seed + 1)
    cache.k_cache.copy_(k)
    cache.v_cache.copy_(v)
    cache.upload_tables()
    return cache, k, v, [list(r) for r in cache.tables]
