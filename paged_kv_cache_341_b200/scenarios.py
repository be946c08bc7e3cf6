"""Set up the synthetic decode workloads on a ``PagedKVCache``.

Blocks come from the library's pool in sequence order s = 0..S-1 (the same
blocks a token-by-token prefill of one sequence after another would take);
K/V values, queries and appended tokens come from the seeded generators in
``workloads``.  ``shared_prefix`` builds 200 sequences that share a
30,720-token prefix (each prefix block referenced 200 times) plus private
suffixes, then forks every sequence once; the decode batch is the 200 forked
children, whose next append copies their shared partly filled last block.
"""

import numpy as np
import torch

from . import workloads
from .cache import PagedKVCache


class Scenario:
    def __init__(self, name, device="cuda", fill_values=True, keep_host=False, block_size=None):
        w = workloads.get(name, block_size)
        self.w = w
        self.lens0 = workloads.lengths(w)
        order = workloads.pool_order(w.num_blocks, w.seed)
        s = w.num_seqs
        rows = 2 * s if w.shared_prefix else s
        self.cache = PagedKVCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.torch_dtype, rows,
                                  w.max_blocks_per_seq, device=device, initial_free_order=order, fill=0.0)
        c = self.cache
        if w.shared_prefix:
            c.allocate(0, w.shared_prefix)
            for r in range(1, s):
                c.share(0, r)
            for r in range(s):
                # private suffix: the table continues after the shared prefix blocks
                first = w.shared_prefix // w.block_size
                need = -(-int(self.lens0[r]) // w.block_size)
                c.tables[r, first:first + need] = c.pool.pa_pool_alloc(need)
                c.lens[r] = w.shared_prefix + int(self.lens0[r])
            for r in range(s):
                c.share(r, s + r)
            self.rows = slice(s, 2 * s)
        else:
            for r in range(s):
                c.allocate(r, int(self.lens0[r]))
            self.rows = slice(0, s)
        self.used_blocks = sorted({int(b) for r in range(rows)
                                   for b in c.tables[r, :-(-int(c.lens[r]) // w.block_size)]})
        self.k_host = self.v_host = None
        if fill_values:
            k, v = workloads.fill_blocks(w, self.used_blocks, w.seed + 100)
            c.k_cache.copy_(k)
            c.v_cache.copy_(v)
            if keep_host:
                self.k_host, self.v_host = k, v
            else:
                del k, v
        c.upload_tables()
        self.step_index = 0

    @property
    def batch(self):
        return self.rows.stop - self.rows.start

    def step_inputs(self, step):
        """Seeded host inputs of decode step ``step``: q [B, Hq, D], k_new/v_new [B, Hkv, D]."""
        seed = self.w.seed + 1000 + 10 * step
        q = workloads.queries(self.w, seed, num_seqs=self.batch)
        k_new, v_new = workloads.new_tokens(self.w, seed + 3, self.batch)
        return q, k_new, v_new

    def kv_bytes(self):
        """Algorithmic K/V bytes one decode step reads: every (token, KV head) row of K and V once."""
        w = self.w
        lens = self.cache.lens[self.rows].astype(np.int64)
        return int(lens.sum()) * 2 * w.num_kv_heads * w.head_dim * w.elem_bytes

    def slot_waste(self):
        """Fraction of allocated token slots left empty in the batch's blocks (tail waste)."""
        w = self.w
        lens = self.cache.lens[self.rows].astype(np.int64)
        blocks = (-(-lens // w.block_size)).sum()
        return float(1.0 - lens.sum() / (blocks * w.block_size))

    def unique_kv_bytes(self):
        """Distinct K/V bytes behind the batch (shared blocks counted once)."""
        w = self.w
        c = self.cache
        seen = set()
        total = 0
        for r in range(self.rows.start, self.rows.stop):
            n = int(c.lens[r])
            for j in range(-(-n // w.block_size)):
                b = int(c.tables[r, j])
                if b in seen:
                    continue
                seen.add(b)
                total += min(w.block_size, n - j * w.block_size)
        return total * 2 * w.num_kv_heads * w.head_dim * w.elem_bytes
