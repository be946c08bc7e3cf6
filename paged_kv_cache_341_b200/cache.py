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

Host-to-device traffic of a step is one small transfer: the slot mapping, the
lengths, the table entries the reservation changed (at most one per row) and
the copy pairs, plus whatever the caller passes from host memory.  The whole
tables go over once, with ``upload_tables``.
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
        # per-step metadata, double-buffered: [slots int64 S][lens int32 S][updates int32 S x 3][pairs int32 S x 2]
        n = max(num_seqs, 1)
        self._meta_bytes = 8 * n + 4 * n + 12 * n + 8 * n
        self._meta_host = [torch.empty(self._meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self._meta_dev = [torch.empty(self._meta_bytes, dtype=torch.uint8, device=self.device) for _ in range(2)]
        self._meta_done = [None, None]    # event: the H2D out of host slot b has finished
        self._meta_views = [self._views(self._meta_host[b]) for b in range(2)]
        self._meta_dviews = [self._views(self._meta_dev[b]) for b in range(2)]
        self._step = 0

    @property
    def num_seqs(self):
        return self.lens.size

    @property
    def step_metadata_bytes(self):
        """Bytes ``decode_step`` sends host -> device besides the caller's tensors."""
        return self._meta_bytes

    def _views(self, buf):
        n = max(self.lens.size, 1)
        o = 0
        slots = buf[o:o + 8 * n].view(torch.int64)
        o += 8 * n
        lens = buf[o:o + 4 * n].view(torch.int32)
        o += 4 * n
        upd = buf[o:o + 12 * n].view(torch.int32).view(n, 3)
        o += 12 * n
        pairs = buf[o:o + 8 * n].view(torch.int32).view(n, 2)
        return slots, lens, upd, pairs

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
        """Reserve one slot in each of ``rows`` (a contiguous range ``slice`` or None = all).

        Works in place on the host tables and lengths (a row range of a
        C-contiguous array is itself contiguous).
        """
        rows = slice(None) if rows is None else rows
        tables = self.tables[rows]
        lens = self.lens[rows]
        assert tables.flags.c_contiguous and lens.flags.c_contiguous
        return self.pool.pa_reserve_slots(tables, lens)

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
        token per row ([B, Hkv, D]); all are CUDA tensors.  The host
        reservation changes at most one table entry per row; those entries,
        the slot mapping, the lengths and the copy pairs go to the device in
        one small transfer, and ``pa_update_block_tables`` applies the entries
        (the device tables must have been uploaded once with
        ``upload_tables``).  Returns the host slot mapping and copy pairs.
        """
        stream = stream or torch.cuda.current_stream()
        sel = slice(None) if rows is None else rows
        r0 = sel.start or 0
        tables = self.tables[sel]
        lens = self.lens[sel]
        assert tables.flags.c_contiguous and lens.flags.c_contiguous
        n = lens.size
        b = self._step & 1
        if self._meta_done[b] is not None:
            self._meta_done[b].synchronize()          # the H2D out of this host slot has finished
        h_slots, h_lens, h_upd, h_pairs = self._meta_views[b]
        d_slots, d_lens, d_upd, d_pairs = self._meta_dviews[b]
        # the reservation writes the slots, pairs and changed table entries straight into the staging
        npairs, nu = self.pool.pa_reserve_slots_with_updates(tables, lens, r0, h_slots.numpy()[:n],
                                                             h_pairs.numpy(), h_upd.numpy())
        self._step += 1
        slots = h_slots.numpy()[:n].copy()
        pairs = h_pairs.numpy()[:npairs].copy()
        h_lens.numpy()[:self.lens.size] = self.lens
        with torch.cuda.stream(stream):
            self._meta_dev[b].copy_(self._meta_host[b], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(stream)
            self._meta_done[b] = ev
        pa.pa_update_block_tables(self.d_tables, d_upd[:nu], self.d_lens, d_lens[:self.lens.size], stream=stream)
        self.copy_blocks(d_pairs[:npairs], stream=stream)
        self.append(k_new, v_new, d_slots[:n], stream=stream)
        self.attend(q, out, scale, partition_size, workspace, tables=self.d_tables[sel], lens=self.d_lens[sel],
                    stream=stream)
        return slots, pairs

    def engine(self, num_q_heads, partition_size=0, stream=None):
        """A native step executor (``pa.Engine``) over this cache's pool, tables and lengths.

        Uploads the tables and lengths first; afterwards steps go through the
        engine (``pa_engine_step``, host buffers in and out).
        """
        self.upload_tables(stream)
        return pa.Engine(self.pool, self.tables, self.lens, self.d_tables, self.d_lens, self.k_cache, self.v_cache,
                         num_q_heads, partition_size, stream)
