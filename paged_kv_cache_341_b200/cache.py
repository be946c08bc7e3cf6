"""A paged KV cache for one attention layer and its decode step.

``PagedKVCache`` owns the host block pool (library pool, FIFO + refcounts),
the host block tables and lengths of a batch of sequences (one row each), and
the device K/V caches ``[num_blocks, block_size, Hkv, D]``.  ``decode_step``
is one pass of the hot path through the C ABI:

1. host: reserve one slot per appending sequence (fresh block at offset 0,
   copy-on-write of a shared partly filled block) -- ``pa_reserve_slots``;
2. device: copy the blocks named by the copy-on-write pairs -- ``pa_copy_blocks``;
3. device: write the new tokens' K/V into their slots -- ``pa_append_kv``;
4. device: single-query attention over every sequence's blocks --
   ``pa_decode_attention`` (split into partitions plus a merge when
   ``partition_size`` > 0).

Host-to-device traffic of a step is the slot mapping, the copy pairs, the
block tables and lengths, plus whatever the caller passes from host memory.
"""

import numpy as np
import torch

from . import pa


class PagedKVCache:
    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim, dtype, num_seqs, max_blocks_per_seq,
                 device="cuda", initial_free_order=None, fill=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self.num_kv_heads = int(num_kv_heads)
        self.head_dim = int(head_dim)
        self.dtype = dtype
        self.device = torch.device(device)
        self.pool = pa.Pool(self.num_blocks, self.block_size, initial_free_order)
        shape = (self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim)
        if fill is None:
            self.k_cache = torch.empty(shape, dtype=dtype, device=self.device)
            self.v_cache = torch.empty(shape, dtype=dtype, device=self.device)
        else:
            self.k_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
            self.v_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
        self.max_blocks = int(max_blocks_per_seq)
        self.tables = np.full((num_seqs, self.max_blocks), -1, np.int32)
        self.lens = np.zeros(num_seqs, np.int32)
        # pinned staging for the per-step host -> device copies
        self._h_tables = torch.empty((num_seqs, self.max_blocks), dtype=torch.int32).pin_memory()
        self._h_lens = torch.empty(num_seqs, dtype=torch.int32).pin_memory()
        self._h_slots = torch.empty(num_seqs, dtype=torch.int64).pin_memory()
        self._h_pairs = torch.empty((max(num_seqs, 1), 2), dtype=torch.int32).pin_memory()
        self.d_tables = torch.empty((num_seqs, self.max_blocks), dtype=torch.int32, device=self.device)
        self.d_lens = torch.empty(num_seqs, dtype=torch.int32, device=self.device)
        self.d_slots = torch.empty(num_seqs, dtype=torch.int64, device=self.device)
        self.d_pairs = torch.empty((max(num_seqs, 1), 2), dtype=torch.int32, device=self.device)
        self._staged = None               # event: last copies out of the pinned staging buffers

    @property
    def num_seqs(self):
        return self.lens.size

    # ---------------------------------------------------------------- host side

    def allocate(self, row, num_tokens):
        """Give row ``row`` (empty) blocks for ``num_tokens`` tokens, front of the free list first."""
        need = -(-int(num_tokens) // self.block_size)
        ids = self.pool.pa_pool_alloc(need)
        self.tables[row, :need] = ids
        self.lens[row] = num_tokens
        return ids

    def share(self, src_row, dst_row):
        """Row ``dst_row`` becomes a sharer of all of ``src_row``'s blocks (fork)."""
        n = -(-int(self.lens[src_row]) // self.block_size)
        self.pool.pa_pool_fork(self.tables[src_row, :n])
        self.tables[dst_row] = self.tables[src_row]
        self.lens[dst_row] = self.lens[src_row]

    def release(self, row):
        n = -(-int(self.lens[row]) // self.block_size)
        self.pool.pa_pool_free(self.tables[row, :n])
        self.tables[row] = -1
        self.lens[row] = 0

    def reserve(self, rows=None):
        """Reserve one slot in each of ``rows`` (a contiguous range ``slice`` or None = all)."""
        rows = slice(None) if rows is None else rows
        tables = np.ascontiguousarray(self.tables[rows])
        lens = np.ascontiguousarray(self.lens[rows])
        slots, pairs = self.pool.pa_reserve_slots(tables, lens)
        self.tables[rows] = tables
        self.lens[rows] = lens
        return slots, pairs

    def _wait_staging(self):
        # the pinned buffers may still be read by an earlier asynchronous copy
        if self._staged is not None:
            self._staged.synchronize()

    def _mark_staging(self, stream):
        self._staged = torch.cuda.Event()
        self._staged.record(stream)

    def upload_tables(self, stream=None):
        """Block tables and lengths to the device (pinned, asynchronous on ``stream``)."""
        stream = stream or torch.cuda.current_stream()
        self._wait_staging()
        self._h_tables.numpy()[:] = self.tables
        self._h_lens.numpy()[:] = self.lens
        with torch.cuda.stream(stream):
            self.d_tables.copy_(self._h_tables, non_blocking=True)
            self.d_lens.copy_(self._h_lens, non_blocking=True)
        self._mark_staging(stream)

    # ------------------------------------------------------------- device side

    def append(self, k_new, v_new, slot_mapping, stream=None):
        pa.pa_append_kv(k_new, v_new, slot_mapping, self.k_cache, self.v_cache, stream=stream)

    def copy_blocks(self, pairs, stream=None):
        if pairs.numel():
            pa.pa_copy_blocks(self.k_cache, self.v_cache, pairs, stream=stream)

    def attend(self, q, out, scale, partition_size=0, workspace=None, tables=None, lens=None, stream=None):
        pa.pa_decode_attention(q, self.k_cache, self.v_cache, self.d_tables if tables is None else tables,
                               self.d_lens if lens is None else lens, scale, out, partition_size=partition_size,
                               workspace=workspace, stream=stream)

    def decode_step(self, q, k_new, v_new, out, scale, partition_size=0, workspace=None, rows=None, stream=None):
        """One decode step for ``rows`` (default all): reserve, copy-on-write, append, attend.

        ``q``/``out`` cover the rows ([B, Hq, D]); ``k_new``/``v_new`` hold one
        token per row ([B, Hkv, D]); all are CUDA tensors.  Returns the host
        slot mapping and copy-on-write pairs of the step.
        """
        stream = stream or torch.cuda.current_stream()
        slots, pairs = self.reserve(rows)
        t = slots.size
        self._wait_staging()
        self._h_slots.numpy()[:t] = slots
        npairs = pairs.shape[0]
        if npairs:
            self._h_pairs.numpy()[:npairs] = pairs
        with torch.cuda.stream(stream):
            self.d_slots[:t].copy_(self._h_slots[:t], non_blocking=True)
            if npairs:
                self.d_pairs[:npairs].copy_(self._h_pairs[:npairs], non_blocking=True)
        self.upload_tables(stream)
        self.copy_blocks(self.d_pairs[:npairs], stream=stream)
        self.append(k_new, v_new, self.d_slots[:t], stream=stream)
        sel = slice(None) if rows is None else rows
        self.attend(q, out, scale, partition_size, workspace, tables=self.d_tables[sel], lens=self.d_lens[sel],
                    stream=stream)
        return slots, pairs
