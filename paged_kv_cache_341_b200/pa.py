"""Python binding of libpagedattn.so (C ABI in include/pa.h).

Argument marshalling only: every step of the decode path runs in the
library's CUDA kernels or its host pool.  Device arguments are torch CUDA
tensors (their ``data_ptr()`` is passed); the stream is torch's current
stream unless one is given.  Importing this module loads the library and
raises ``ImportError`` when it has not been built -- there is no fallback.

Function names match the C entry points.
"""

import ctypes
import os

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        "libpagedattn.so is not built (expected at %s); run `python -m paged_kv_cache_341_b200.build`" % _LIB_PATH)
_lib = ctypes.CDLL(_LIB_PATH)

PA_OK, PA_ERR_EXHAUSTED, PA_ERR_INVALID, PA_ERR_REFCOUNT, PA_ERR_CUDA, PA_ERR_DEVICE_CHECK, PA_ERR_UNSUPPORTED = range(7)
PA_F32, PA_F16, PA_BF16 = 0, 1, 2
DTYPE_CODE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}

# Every symbol include/pa.h declares, with its C signature.
_i32, _i64, _sz, _vp, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
_p32 = ctypes.POINTER(ctypes.c_int32)
_p64 = ctypes.POINTER(ctypes.c_int64)
SIGNATURES = {
    "pa_pool_create": (_i32, [_i32, _i32, _p32, ctypes.POINTER(_vp)]),
    "pa_pool_destroy": (None, [_vp]),
    "pa_pool_alloc": (_i32, [_vp, _i32, _p32]),
    "pa_pool_free": (_i32, [_vp, _p32, _i32]),
    "pa_pool_fork": (_i32, [_vp, _p32, _i32]),
    "pa_pool_refcount": (_i32, [_vp, _i32, _p32]),
    "pa_pool_num_free": (_i32, [_vp, _p32]),
    "pa_pool_export": (_i32, [_vp, _p32, _p32, _p32]),
    "pa_seq_reserve_slot": (_i32, [_vp, _p32, _i32, _p32, _p64, _p32, _p32]),
    "pa_reserve_slots": (_i32, [_vp, _p32, _i32, _p32, _i32, _p64, _p32, _p32]),
    "pa_reserve_slots_with_updates": (_i32, [_vp, _p32, _i32, _p32, _i32, _i32, _p64, _p32, _p32, _p32, _p32]),
    "pa_pool_enable_prefix_cache": (_i32, [_vp]),
    "pa_seq_alloc_prompt": (_i32, [_vp, _p32, _i32, _p32, _i32, _p32]),
    "pa_pool_cached_blocks": (_i32, [_vp, _p32]),
    "pa_prefix_hash": (_i32, [_p32, _i32, ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint64)]),
    "pa_append_kv": (_i32, [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pa_copy_blocks": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pa_update_block_tables": (_i32, [_vp, _i32, _i32, _vp, _i32, _vp, _vp, _i32, _vp]),
    "pa_read_stream": (_i32, [_vp, _sz, _vp, _vp]),
    "pa_engine_create": (_i32, [_vp, _p32, _p32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                ctypes.POINTER(_vp)]),
    "pa_engine_destroy": (None, [_vp]),
    "pa_engine_step": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _f32, _p64, _p32, _p32]),
    "pa_engine_join": (_i32, [_vp]),
    "pa_engine_synchronize": (_i32, [_vp]),
    "pa_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "pa_decode_attention": (_i32, [_vp, _vp, _vp, _i32, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _i32,
                                   _vp, _sz, _vp, _i32, _vp]),
    "pa_decode_attention_static": (_i32, [_vp, _vp, _vp, _i32, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _f32,
                                          _i32, _vp, _i32, _vp]),
    "pa_shared_prefix_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pa_decode_attention_shared_prefix": (_i32, [_vp, _vp, _vp, _i32, _vp, _i32, _vp, _i32, _i32, _vp, _i32, _i32,
                                                 _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp, _i32, _vp]),
    "pa_device_error": (_i32, [_p32, _i32]),
    "pa_debug_decode_stall": (_i32, [_i64]),
    "pa_debug_last_prefix_kernel": (_i32, []),
    "pa_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class PagedAttnError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("status %d: %s" % (status, message))
        self.status = status


class PoolExhausted(PagedAttnError):
    """No free block is left (the pages' "KV cache exhausted")."""


def library_path():
    return _LIB_PATH


def pa_last_error():
    return _lib.pa_last_error().decode()


def _check(status):
    if status != PA_OK:
        cls = PoolExhausted if status == PA_ERR_EXHAUSTED else PagedAttnError
        raise cls(status, pa_last_error())


def _i32_array(values):
    arr = np.ascontiguousarray(np.asarray(values, dtype=np.int32))
    return arr, arr.ctypes.data_as(_p32)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t, name, dtype=None):
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must have dtype %s, got %s" % (name, dtype, t.dtype))
    return ctypes.c_void_p(t.data_ptr())


# --------------------------------------------------------------------------
# Host block pool
# --------------------------------------------------------------------------

class Pool:
    """Refcounted block pool (pa_pool_*).  Host memory only; not thread-safe."""

    def __init__(self, num_blocks, block_size, initial_free_order=None):
        handle = ctypes.c_void_p()
        if initial_free_order is None:
            _check(_lib.pa_pool_create(num_blocks, block_size, None, ctypes.byref(handle)))
        else:
            arr, ptr = _i32_array(initial_free_order)
            if arr.size != num_blocks:
                raise ValueError("initial_free_order must have num_blocks entries")
            _check(_lib.pa_pool_create(num_blocks, block_size, ptr, ctypes.byref(handle)))
        self._h = handle
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            _lib.pa_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def pa_pool_alloc(self, n):
        out = np.empty(max(n, 0), np.int32)
        _check(_lib.pa_pool_alloc(self._h, n, out.ctypes.data_as(_p32)))
        return out

    def pa_pool_free(self, ids):
        arr, ptr = _i32_array(ids)
        _check(_lib.pa_pool_free(self._h, ptr, arr.size))

    def pa_pool_fork(self, ids):
        arr, ptr = _i32_array(ids)
        _check(_lib.pa_pool_fork(self._h, ptr, arr.size))

    def pa_pool_refcount(self, block_id):
        out = ctypes.c_int32()
        _check(_lib.pa_pool_refcount(self._h, block_id, ctypes.byref(out)))
        return out.value

    def pa_pool_num_free(self):
        out = ctypes.c_int32()
        _check(_lib.pa_pool_num_free(self._h, ctypes.byref(out)))
        return out.value

    def pa_pool_export(self):
        refs = np.empty(self.num_blocks, np.int32)
        free = np.empty(self.num_blocks, np.int32)
        n = ctypes.c_int32()
        _check(_lib.pa_pool_export(self._h, refs.ctypes.data_as(_p32), free.ctypes.data_as(_p32), ctypes.byref(n)))
        return refs, free[: n.value].copy()

    def pa_seq_reserve_slot(self, table, length):
        """``table``: writable int32 numpy array (the sequence's row).  Returns (slot, new_len, src, dst)."""
        if table.dtype != np.int32 or not table.flags.c_contiguous:
            raise TypeError("table must be a contiguous int32 array")
        n = ctypes.c_int32(length)
        slot = ctypes.c_int64()
        src, dst = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.pa_seq_reserve_slot(self._h, table.ctypes.data_as(_p32), table.size, ctypes.byref(n),
                                        ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)))
        return slot.value, n.value, src.value, dst.value

    def pa_reserve_slots(self, tables, lens):
        """One step for every row of ``tables`` ([S, cap] int32, in place) and ``lens`` ([S] int32, in place).

        Returns (slots int64 [S], pairs int32 [P, 2]).
        """
        if tables.dtype != np.int32 or lens.dtype != np.int32 or not tables.flags.c_contiguous:
            raise TypeError("tables and lens must be contiguous int32 arrays")
        s = lens.size
        slots = np.empty(s, np.int64)
        pairs = np.empty((max(s, 1), 2), np.int32)
        npairs = ctypes.c_int32()
        _check(_lib.pa_reserve_slots(self._h, tables.ctypes.data_as(_p32), tables.shape[1],
                                     lens.ctypes.data_as(_p32), s, slots.ctypes.data_as(_p64),
                                     pairs.ctypes.data_as(_p32), ctypes.byref(npairs)))
        return slots, pairs[: npairs.value].copy()

    def pa_reserve_slots_with_updates(self, tables, lens, row0, slots_out, pairs_out, updates_out):
        """``pa_reserve_slots`` writing into caller arrays, also listing the table entries it wrote.

        ``slots_out`` int64 [S], ``pairs_out`` int32 [>=S, 2], ``updates_out`` int32 [>=S, 3] (each
        contiguous, e.g. views of pinned staging); returns (number of pairs, number of updates).
        """
        if tables.dtype != np.int32 or lens.dtype != np.int32 or not tables.flags.c_contiguous:
            raise TypeError("tables and lens must be contiguous int32 arrays")
        s = lens.size
        for a, dt, w in ((slots_out, np.int64, 1), (pairs_out, np.int32, 2), (updates_out, np.int32, 3)):
            if a.dtype != dt or not a.flags.c_contiguous or a.size < w * s:
                raise TypeError("output arrays: contiguous, of the right type and size")
        npairs, nupd = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.pa_reserve_slots_with_updates(self._h, tables.ctypes.data_as(_p32), tables.shape[1],
                                                  lens.ctypes.data_as(_p32), s, int(row0),
                                                  slots_out.ctypes.data_as(_p64), pairs_out.ctypes.data_as(_p32),
                                                  ctypes.byref(npairs), updates_out.ctypes.data_as(_p32),
                                                  ctypes.byref(nupd)))
        return npairs.value, nupd.value


    # -- prefix caching ------------------------------------------------------

    def pa_pool_enable_prefix_cache(self):
        _check(_lib.pa_pool_enable_prefix_cache(self._h))

    def pa_seq_alloc_prompt(self, tokens, table):
        """Blocks for a prompt (``table``: writable int32 array); returns the number of cached tokens."""
        arr, ptr = _i32_array(tokens)
        if table.dtype != np.int32 or not table.flags.c_contiguous:
            raise TypeError("table must be a contiguous int32 array")
        cached = ctypes.c_int32()
        _check(_lib.pa_seq_alloc_prompt(self._h, ptr, arr.size, table.ctypes.data_as(_p32), table.size,
                                        ctypes.byref(cached)))
        return cached.value

    def pa_pool_cached_blocks(self):
        out = ctypes.c_int32()
        _check(_lib.pa_pool_cached_blocks(self._h, ctypes.byref(out)))
        return out.value


def pa_prefix_hash(tokens, seed=0):
    arr, ptr = _i32_array(tokens)
    out = ctypes.c_uint64()
    _check(_lib.pa_prefix_hash(ptr, arr.size, seed, ctypes.byref(out)))
    return out.value


# --------------------------------------------------------------------------
# Device kernels
# --------------------------------------------------------------------------

def pa_append_kv(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None):
    """k_new/v_new [T, Hkv, D], slot_mapping int64 [T] (CUDA), caches [NB, bs, Hkv, D]."""
    nb, bs, hkv, d = k_cache.shape
    code = DTYPE_CODE[k_cache.dtype]
    _check(_lib.pa_append_kv(_dev(k_new, "k_new", k_cache.dtype), _dev(v_new, "v_new", k_cache.dtype),
                             _dev(slot_mapping, "slot_mapping", torch.int64), slot_mapping.numel(),
                             _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype), nb, bs, hkv, d, code,
                             _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, pairs, stream=None):
    """pairs: int32 CUDA tensor [P, 2] of (src, dst) block ids."""
    nb, bs, hkv, d = k_cache.shape
    code = DTYPE_CODE[k_cache.dtype]
    _check(_lib.pa_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype),
                               _dev(pairs, "pairs", torch.int32), pairs.shape[0] if pairs.numel() else 0, nb, bs, hkv,
                               d, code, _stream(stream)))


def pa_update_block_tables(block_tables, updates, context_lens=None, new_lens=None, stream=None):
    """block_tables: int32 CUDA [rows, stride] (row-contiguous); updates: int32 CUDA [n, 3] (row, column, id).

    With ``context_lens`` (int32 CUDA [rows]) the same launch also sets
    ``context_lens[:len(new_lens)] = new_lens``.
    """
    if block_tables.dim() != 2 or block_tables.stride(1) != 1:
        raise ValueError("block_tables must be a 2-D tensor with unit column stride")
    n = updates.shape[0] if updates.numel() else 0
    nl = 0 if context_lens is None else new_lens.numel()
    _check(_lib.pa_update_block_tables(ctypes.c_void_p(block_tables.data_ptr()), block_tables.shape[0],
                                       block_tables.stride(0), _dev(updates, "updates", torch.int32) if n else None,
                                       n, _dev(context_lens, "context_lens", torch.int32) if nl else None,
                                       _dev(new_lens, "new_lens", torch.int32) if nl else None, nl, _stream(stream)))


def pa_read_stream(buf, sink, stream=None):
    """Read all of ``buf`` (CUDA tensor, contiguous) once; XOR of what was read lands in ``sink`` (int32 CUDA [1])."""
    _check(_lib.pa_read_stream(_dev(buf, "buf"), buf.numel() * buf.element_size(), _dev(sink, "sink", torch.int32),
                               _stream(stream)))


def pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size, partition_size):
    return int(_lib.pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size,
                                             partition_size))


def decode_workspace(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size, partition_size, device=None):
    """Allocate (through torch) the workspace pa_decode_attention needs; None when none is needed."""
    nbytes = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size, partition_size)
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def pa_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale, out, partition_size=0,
                        workspace=None, stream=None):
    """q, out [S, Hq, D]; caches [NB, bs, Hkv, D]; block_tables int32 [S, MB]; context_lens int32 [S]."""
    s, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(out.shape) != (s, hq, d):
        raise ValueError("shape mismatch between q, caches and out")
    code = DTYPE_CODE[k_cache.dtype]
    ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode_attention(_dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
                                    _dev(v_cache, "v_cache", k_cache.dtype), nb,
                                    _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                                    _dev(context_lens, "context_lens", torch.int32), s, hq, hkv, d, bs, float(scale),
                                    int(partition_size), ws_ptr, ws_bytes, _dev(out, "out", k_cache.dtype), code,
                                    _stream(stream)))


def pa_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim, prefix_len, max_suffix_blocks, block_size,
                                    partition_size):
    return int(_lib.pa_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim, prefix_len, max_suffix_blocks,
                                                    block_size, partition_size))


def pa_decode_attention_shared_prefix(q, k_cache, v_cache, prefix_blocks, prefix_len, suffix_tables, suffix_lens,
                                      scale, out, partition_size=0, workspace=None, stream=None):
    """Decode attention over a prefix shared by every sequence followed by each sequence's own suffix.

    prefix_blocks: int32 CUDA [prefix_len / block_size]; suffix_tables: int32 CUDA [S, >= max suffix blocks]
    (a row-slice view of a wider table is fine: its row stride is passed); suffix_lens: int32 CUDA [S].
    The workspace (pa_shared_prefix_workspace_size bytes) is allocated here through torch when not given.
    """
    s, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(out.shape) != (s, hq, d):
        raise ValueError("shape mismatch between q, caches and out")
    if suffix_tables.dim() != 2 or suffix_tables.stride(1) != 1:
        raise ValueError("suffix_tables must be a 2-D tensor with unit column stride")
    if suffix_tables.dtype != torch.int32 or not suffix_tables.is_cuda:
        raise TypeError("suffix_tables must be an int32 CUDA tensor")
    max_suffix = suffix_tables.shape[1]
    if workspace is None:
        nbytes = pa_shared_prefix_workspace_size(s, hq, d, int(prefix_len), max_suffix, bs, int(partition_size))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    code = DTYPE_CODE[k_cache.dtype]
    pb = _dev(prefix_blocks, "prefix_blocks", torch.int32) if int(prefix_len) > 0 else None
    _check(_lib.pa_decode_attention_shared_prefix(
        _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype), nb,
        pb, int(prefix_len), ctypes.c_void_p(suffix_tables.data_ptr()), suffix_tables.stride(0), max_suffix,
        _dev(suffix_lens, "suffix_lens", torch.int32), s, hq, hkv, d, bs, float(scale), int(partition_size),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(),
        _dev(out, "out", k_cache.dtype), code, _stream(stream)))
    return workspace


STATIC_WORKSPACE_BYTES = 32 * 1024 * 1024


def pa_decode_attention_static(q, k_cache, v_cache, block_tables, context_lens, scale, out, partition_size=0,
                               stream=None):
    """pa_decode_attention with no workspace argument, for callers that cannot allocate device memory.

    The split-context partials go to a static 32 MiB device array inside the
    library (shared by every call on the device; overlapping calls race), so
    nothing is allocated here or in the library.  Sizes whose workspace would
    exceed 32 MiB are rejected.  The first call on a device looks the array up
    and should come before any stream capture.
    """
    s, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(out.shape) != (s, hq, d):
        raise ValueError("shape mismatch between q, caches and out")
    code = DTYPE_CODE[k_cache.dtype]
    _check(_lib.pa_decode_attention_static(_dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
                                           _dev(v_cache, "v_cache", k_cache.dtype), nb,
                                           _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                                           _dev(context_lens, "context_lens", torch.int32), s, hq, hkv, d, bs,
                                           float(scale), int(partition_size), _dev(out, "out", k_cache.dtype), code,
                                           _stream(stream)))


def pa_device_error(reset=True):
    """Synchronise and return the device error word (0 = no bad index seen)."""
    code = ctypes.c_int32()
    _check(_lib.pa_device_error(ctypes.byref(code), 1 if reset else 0))
    return code.value


def pa_debug_last_prefix_kernel():
    """1 = SM-pair tcgen05 prefix kernel, 2 = one-SM tcgen05, 3 = mma.sync, 0 = none yet (this thread)."""
    return int(_lib.pa_debug_last_prefix_kernel())


def pa_debug_decode_stall(wait_limit_ns):
    """Test hook of the bounded waits (0 = off): see include/pa.h."""
    _check(_lib.pa_debug_decode_stall(int(wait_limit_ns)))


# --------------------------------------------------------------------------
# Step executor
# --------------------------------------------------------------------------

def _host(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError("%s must be a host (CPU) tensor" % name)
    if not t.is_contiguous() or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError("%s must be a contiguous %s tensor of shape %s" % (name, dtype, tuple(shape)))
    return ctypes.c_void_p(t.data_ptr())


class Engine:
    """pa_engine_*: one decode step of a batch per call, host buffers in and out.

    ``host_tables`` / ``host_lens`` are the caller's numpy int32 arrays
    ([S, max_blocks], [S]), changed in place by every step; ``device_tables``
    / ``device_lens`` their CUDA copies (already uploaded).  The engine keeps
    references to all of them so they outlive it.
    """

    def __init__(self, pool, host_tables, host_lens, device_tables, device_lens, k_cache, v_cache, num_q_heads,
                 partition_size=0, stream=None):
        if host_tables.dtype != np.int32 or not host_tables.flags.c_contiguous or host_tables.ndim != 2:
            raise TypeError("host_tables must be a C-contiguous int32 [S, max_blocks] array")
        if host_lens.dtype != np.int32 or not host_lens.flags.c_contiguous or host_lens.size != host_tables.shape[0]:
            raise TypeError("host_lens must be a contiguous int32 [S] array")
        nb, bs, hkv, d = k_cache.shape
        s, mb = host_tables.shape
        if tuple(device_tables.shape) != (s, mb) or device_lens.numel() != s:
            raise ValueError("device tables/lengths must match the host ones")
        self._keep = (pool, host_tables, host_lens, device_tables, device_lens, k_cache, v_cache)
        self._stream = stream if stream is not None else torch.cuda.current_stream()
        self.dtype = k_cache.dtype
        self.num_q_heads, self.num_kv_heads, self.head_dim = num_q_heads, hkv, d
        handle = ctypes.c_void_p()
        _check(_lib.pa_engine_create(pool._h, host_tables.ctypes.data_as(_p32), host_lens.ctypes.data_as(_p32), s,
                                     mb, _dev(device_tables, "device_tables", torch.int32),
                                     _dev(device_lens, "device_lens", torch.int32), _dev(k_cache, "k_cache"),
                                     _dev(v_cache, "v_cache", k_cache.dtype), num_q_heads, hkv, d,
                                     DTYPE_CODE[k_cache.dtype], partition_size, _stream(self._stream),
                                     ctypes.byref(handle)))
        self._h = handle
        self._slots = np.empty(s, np.int64)
        self._pairs = np.empty((s, 2), np.int32)

    def close(self):
        if getattr(self, "_h", None):
            _lib.pa_engine_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def pa_engine_step(self, row0, num_rows, q, k_new, v_new, out, scale, want_slots=False):
        """Enqueue one step; returns (slots, pairs) copies when ``want_slots`` else the pair count."""
        hq, hkv, d = self.num_q_heads, self.num_kv_heads, self.head_dim
        npairs = ctypes.c_int32()
        _check(_lib.pa_engine_step(self._h, row0, num_rows, _host(q, "q", self.dtype, (num_rows, hq, d)),
                                   _host(k_new, "k_new", self.dtype, (num_rows, hkv, d)),
                                   _host(v_new, "v_new", self.dtype, (num_rows, hkv, d)),
                                   _host(out, "out", self.dtype, (num_rows, hq, d)), scale,
                                   self._slots.ctypes.data_as(_p64) if want_slots else None,
                                   self._pairs.ctypes.data_as(_p32) if want_slots else None, ctypes.byref(npairs)))
        if want_slots:
            return self._slots[:num_rows].copy(), self._pairs[:npairs.value].copy()
        return npairs.value

    def pa_engine_join(self):
        _check(_lib.pa_engine_join(self._h))

    def pa_engine_synchronize(self):
        _check(_lib.pa_engine_synchronize(self._h))
