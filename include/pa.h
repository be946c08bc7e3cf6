/*
 * pa.h -- C ABI of libpagedattn.so, a paged KV cache decode path for NVIDIA
 * B200 (sm_100a).
 *
 * What it implements, from the descriptions of PagedAttention on four web
 * pages (no code from them is used):
 *
 *   - a pool of equally sized physical KV blocks that each sequence reaches
 *     through its own block table ("PagedAttention Explained: Managing KV Cache
 *     Efficiently", agentechip.com, section "Block Tables and Non-Contiguous
 *     Storage"; "Master Paged Attention for LLM Inference", krapton.com,
 *     section "How Paged Attention Works: The Mechanics", steps 1-3);
 *   - blocks handed out on demand from a first-in first-out free list, with a
 *     reference count per block, and copy-on-write for blocks that several
 *     sequences share (agentechip.com, sections "Implementing a Simplified
 *     Paged KV Cache" and "Shared Prefix Caching"; krapton.com step 4);
 *   - the device kernels of one decode step: copy of shared blocks before a
 *     write, append of the new token's K/V into its slot, and single-query
 *     attention that walks the block table instead of gathering the blocks
 *     (agentechip.com, "Block Tables and Non-Contiguous Storage" and the
 *     closing remark of "Implementing a Simplified Paged KV Cache").
 *
 * Conventions for every call:
 *   - Status codes only; nothing throws, aborts or traps.  On failure,
 *     pa_last_error() returns a message (per calling thread).
 *   - Only pa_engine_create allocates (its own device staging, page-locked
 *     host staging, streams and events, all freed by pa_engine_destroy); no
 *     other call allocates device memory.  Caches, tables, workspace and
 *     outputs are device buffers owned by the caller (e.g. torch tensors'
 *     data_ptr()).  Host arrays are owned by the caller too.
 *   - Device calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and only enqueue work.  A launch failure returns
 *     PA_ERR_CUDA.  Bad indices found on the device (a block id outside the
 *     pool, a slot outside the cache, a length beyond the table) never fault:
 *     the access is skipped or clamped and a device error word is set, which
 *     pa_device_error() reads after the stream is synchronised.
 *   - Cache layout, K and V alike: [num_blocks][block_size][num_kv_heads]
 *     [head_dim], contiguous, element type `dtype` -- each block holds
 *     block_size token rows of (num_kv_heads, head_dim), the per-block shape of
 *     the toy cache in agentechip.com "Implementing a Simplified Paged KV
 *     Cache".  Device pointers must be 16-byte aligned.
 *   - A flat slot index x names block x / block_size, row x % block_size.
 */
#ifndef PAGEDATTN_PA_H
#define PAGEDATTN_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_EXHAUSTED = 1,     /* no free block: the pages' "KV cache exhausted"   */
  PA_ERR_INVALID = 2,       /* bad argument (range, size, alignment, null)      */
  PA_ERR_REFCOUNT = 3,      /* release/share not allowed by the reference count */
  PA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed             */
  PA_ERR_DEVICE_CHECK = 5,  /* a kernel found a bad index (see pa_device_error) */
  PA_ERR_UNSUPPORTED = 6    /* shape/dtype combination not compiled in          */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* ------------------------------------------------------------------------ */
/* Host block pool.  Opaque, host memory only, not thread-safe.             */
/* Every failing call leaves the pool unchanged (all or nothing).           */
/* ------------------------------------------------------------------------ */
typedef struct pa_pool pa_pool;

/* Create a pool of `num_blocks` blocks of `block_size` tokens.  The free list
 * starts as `initial_free_order` (a permutation of 0..num_blocks-1, copied),
 * or as 0..num_blocks-1 when it is NULL (the toy pool's starting list in
 * agentechip.com "Implementing a Simplified Paged KV Cache").
 * Errors: PA_ERR_INVALID (num_blocks < 0, block_size <= 0, not a permutation,
 * out == NULL). */
pa_status pa_pool_create(int32_t num_blocks, int32_t block_size,
                         const int32_t* initial_free_order, pa_pool** out);
void pa_pool_destroy(pa_pool* pool);

/* Take `n` blocks from the FRONT of the free list into out_ids[0..n), each
 * with reference count 1.  Errors: PA_ERR_EXHAUSTED if fewer than n are
 * free; PA_ERR_INVALID for n < 0 or a NULL buffer with n > 0. */
pa_status pa_pool_alloc(pa_pool* pool, int32_t n, int32_t* out_ids);

/* Drop one reference per listed id (duplicates count twice); a block whose
 * count reaches 0 goes to the BACK of the free list, in list order
 * (agentechip.com "Implementing a Simplified Paged KV Cache").  Errors:
 * PA_ERR_INVALID (id out of range), PA_ERR_REFCOUNT (more releases than
 * references). */
pa_status pa_pool_free(pa_pool* pool, const int32_t* ids, int32_t n);

/* Add one reference per listed id: a second sequence now shares the block
 * (copy-on-write sharing, krapton.com step 4 "Shared Blocks").  The caller
 * copies the parent's table and length for the child.  Errors:
 * PA_ERR_INVALID (id out of range), PA_ERR_REFCOUNT (block is free). */
pa_status pa_pool_fork(pa_pool* pool, const int32_t* ids, int32_t n);

pa_status pa_pool_refcount(const pa_pool* pool, int32_t id, int32_t* out);
pa_status pa_pool_num_free(const pa_pool* pool, int32_t* out);

/* Copy the state out: refcounts[num_blocks] by block id, free_list[n_free]
 * front to back (buffer of num_blocks entries). */
pa_status pa_pool_export(const pa_pool* pool, int32_t* refcounts, int32_t* free_list,
                         int32_t* n_free);

/* Reserve the slot of token number *len of one sequence and advance *len.
 * `table` is the sequence's host block table with room for `table_cap`
 * entries.  Offset 0 of a block takes a fresh block from the free list.  At
 * offset > 0, when the current block's count is above 1 (shared), the
 * sequence moves to a fresh block: the old block loses one reference, the
 * table entry changes, and (*cow_src_out, *cow_dst_out) name the copy the
 * caller must run (pa_copy_blocks) before appending; otherwise both are -1.
 * The plainest reading of "copy-on-write" on the pages (agentechip.com
 * "Shared Prefix Caching"), which give no trigger rule of their own.
 * Errors: PA_ERR_EXHAUSTED (no block for a new block or a copy),
 * PA_ERR_INVALID (table too small, table entry free or out of range). */
pa_status pa_seq_reserve_slot(pa_pool* pool, int32_t* table, int32_t table_cap, int32_t* len,
                              int64_t* slot_out, int32_t* cow_src_out, int32_t* cow_dst_out);

/* One decode step's reservations for S sequences, in order s = 0..S-1:
 * pa_seq_reserve_slot on row s of `tables` ([S][table_cap], host) with
 * lens[s]; slots_out[s] receives the slot; every copy-on-write pair is
 * appended to pairs_out ([S][2] room) and counted in *num_pairs_out.  All or
 * nothing: on any failure the pool, tables and lens are restored. */
pa_status pa_reserve_slots(pa_pool* pool, int32_t* tables, int32_t table_cap, int32_t* lens,
                           int32_t num_seqs, int64_t* slots_out, int32_t* pairs_out,
                           int32_t* num_pairs_out);

/* pa_reserve_slots that also lists the block-table entries the step wrote,
 * for a caller that keeps a device copy of the tables up to date without
 * re-sending them: updates_out ([S][3] room, host) receives one
 * (row0 + s, column, block id) triple for every sequence s whose reserved
 * token took a block -- a fresh block at offset 0, or the private copy of a
 * shared block -- and *num_updates_out their count.  These are exactly the
 * entries to pass to pa_update_block_tables.  updates_out may be NULL (then
 * this is pa_reserve_slots).  All or nothing, as pa_reserve_slots. */
pa_status pa_reserve_slots_with_updates(pa_pool* pool, int32_t* tables, int32_t table_cap, int32_t* lens,
                                        int32_t num_seqs, int32_t row0, int64_t* slots_out,
                                        int32_t* pairs_out, int32_t* num_pairs_out,
                                        int32_t* updates_out, int32_t* num_updates_out);

/* Prefix caching by block content ("Paged Attention", aidolsgroup.com, "Why
 * it matters": every KV-cache block is hashed by its tokens and the tokens
 * before it, so requests sharing a system prompt reuse the same blocks).
 * Key of full block i of a prompt: 64-bit FNV-1a over the little-endian bytes
 * of the int32 token ids tokens[0 : (i+1)*block_size].  Only full blocks are
 * registered; a block leaves the cache when it returns to the free list. */
pa_status pa_pool_enable_prefix_cache(pa_pool* pool);

/* Blocks for a new sequence holding the prompt tokens[0..num_tokens): the
 * leading full blocks whose key is registered (and whose stored token ids
 * match) are shared (reference count + 1); the search stops at the first
 * miss; the remaining blocks come from the front of the free list and each new
 * full block is registered unless its key already is.  table[0 ..
 * ceil(num_tokens/block_size)) receives the blocks; *num_cached_tokens the
 * tokens whose K/V are already present (a multiple of block_size) -- the
 * caller writes K/V for the rest.  All or nothing.  Errors: PA_ERR_EXHAUSTED,
 * PA_ERR_INVALID (cache not enabled, table too small, bad argument). */
pa_status pa_seq_alloc_prompt(pa_pool* pool, const int32_t* tokens, int32_t num_tokens, int32_t* table,
                              int32_t table_cap, int32_t* num_cached_tokens);

/* Number of blocks currently findable by key. */
pa_status pa_pool_cached_blocks(const pa_pool* pool, int32_t* out);

/* The key function itself: FNV-1a 64 of tokens[0..num_tokens) continued from
 * `seed` (0 = the FNV offset basis). */
pa_status pa_prefix_hash(const int32_t* tokens, int32_t num_tokens, uint64_t seed, uint64_t* out);

/* ------------------------------------------------------------------------ */
/* Device kernels (sm_100a).                                                */
/* ------------------------------------------------------------------------ */

/* Append: for t < T with slot_mapping[t] >= 0, write k_new[t] ([Hkv][D]) and
 * v_new[t] into row slot % block_size of block slot / block_size (the write of
 * a new token into its block, agentechip.com "Implementing a Simplified Paged
 * KV Cache").  k_new, v_new: device [T][Hkv][D]; slot_mapping: device int64
 * [T]; slots must be distinct.  A slot >= num_blocks*block_size is skipped and
 * sets the device error word.  Bit copy. */
pa_status pa_append_kv(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                       int32_t num_tokens, void* k_cache, void* v_cache, int32_t num_blocks,
                       int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                       pa_dtype dtype, void* stream);

/* Copy-on-write block copy: for each pair p, K and V block pairs[p][1] become
 * bit copies of block pairs[p][0] (krapton.com step 4; agentechip.com
 * "Shared Prefix Caching").  pairs: device int32 [P][2]; destinations must be
 * distinct and no destination may also be a source in the same call.  Ids
 * outside [0, num_blocks) are skipped and set the device error word. */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t num_pairs,
                         int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                         int32_t head_dim, pa_dtype dtype, void* stream);

/* Write changed block-table entries on the device: updates is a device int32
 * [num_updates][3] array of (row, column, block id), applied to
 * block_tables (device int32 [num_rows][table_stride]).  A host reservation
 * changes at most one entry per appending sequence (a fresh block at a block
 * boundary, or the private copy of a shared block), so sending the changes
 * instead of the tables keeps a step's host-to-device traffic small.
 * Out-of-range rows or columns are skipped and set the device error word (3).
 * Entries with the same (row, column) in one call must not repeat.
 * When context_lens (device int32 [num_rows]) is non-NULL, the same launch
 * sets context_lens[i] = new_lens[i] for i < num_lens (device int32 array,
 * num_lens <= num_rows); NULL context_lens skips the lengths. */
pa_status pa_update_block_tables(int32_t* block_tables, int32_t num_rows, int32_t table_stride,
                                 const int32_t* updates, int32_t num_updates, int32_t* context_lens,
                                 const int32_t* new_lens, int32_t num_lens, void* stream);

/* Bytes of device workspace pa_decode_attention takes for these sizes: 256
 * bytes for the work-unit counter, a planned work-unit list of 16 bytes per
 * (sequence, query head, partition) rounded up to 256 bytes, plus, when
 * partition_size > 0, one float32 partial (max, sum, D values) per (sequence,
 * query head, partition); partitions = ceil(max_blocks_per_seq * block_size /
 * partition_size), or 1 when partition_size == 0.  0 for invalid sizes. */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_blocks_per_seq, int32_t block_size,
                                int32_t partition_size);

/* Single-query decode attention over the paged cache.  For every sequence s
 * and query head h, with kv = h / (Hq / Hkv):
 *   out[s][h] = softmax_j(q[s][h] . K_s[j][kv] * scale) V_s[j][kv],
 *   j < context_lens[s], where K_s[j] is row j % block_size of block
 *   block_tables[s][j / block_size] (and V likewise).
 * That is ordinary attention over the sequence's tokens in logical order: the
 * kernel walks the block table and never gathers the blocks
 * (agentechip.com "Block Tables and Non-Contiguous Storage"; krapton.com
 * "FAQ": paging leaves the computation unchanged).  Accumulation is float32
 * (online softmax with a running maximum and sum).  Grouped query heads
 * (Hq > Hkv) share every K/V load.  context_lens[s] == 0 writes a zero row.
 *
 *   q, out:        device [S][Hq][D], element type dtype (out rounded to
 *                  nearest even from float32)
 *   k/v_cache:     device [num_blocks][block_size][Hkv][D]
 *   block_tables:  device int32 [S][max_blocks_per_seq]; entries that cover
 *                  tokens < context_lens[s] must be valid block ids
 *   context_lens:  device int32 [S], each <= max_blocks_per_seq*block_size
 *   partition_size 0: one pass over each whole context.  > 0 (a multiple of
 *                  block_size and of 16): split each context into partitions of
 *                  that many tokens, compute partial (max, sum, output) per
 *                  partition and merge them with a second kernel (launched
 *                  as a programmatic dependent of the first).
 *   workspace      device buffer of pa_decode_workspace_size() bytes, owned
 *                  by the caller; required when partition_size > 0.  With a
 *                  workspace, a one-CTA planning kernel first lists the work
 *                  units in it (full partitions, then the rest longest first)
 *                  and the decode kernel takes them through a counter; with
 *                  NULL (only when partition_size == 0) the units are dealt
 *                  round-robin.  Calls sharing a workspace must not
 *                  overlap on the GPU.
 * Supported: head_dim 64 or 128; Hq/Hkv in {1,2,4,8}; block_size a multiple
 * of 16, or 8; dtype f32/f16/bf16.  Errors: PA_ERR_INVALID, PA_ERR_UNSUPPORTED,
 * PA_ERR_CUDA. */
pa_status pa_decode_attention(const void* q, const void* k_cache, const void* v_cache,
                              int32_t num_blocks, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* context_lens,
                              int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, float scale,
                              int32_t partition_size, void* workspace, size_t workspace_bytes,
                              void* out, pa_dtype dtype, void* stream);

/* Bytes of device workspace pa_decode_attention_shared_prefix takes: 256
 * bytes for the work-unit counter, the suffix's work-unit list (as for
 * pa_decode_workspace_size) and one float32 partial (max, sum, D values) per
 * (sequence, query head, part), where the parts are the prefix's
 * ceil(prefix_len / 512) slices followed by the suffix's partitions
 * (ceil(max_suffix_blocks * block_size / partition_size), or 1 when
 * partition_size == 0).  0 for invalid sizes. */
size_t pa_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                       int32_t prefix_len, int32_t max_suffix_blocks,
                                       int32_t block_size, int32_t partition_size);

/* Decode attention when every sequence starts with the same prefix blocks
 * (a system prompt shared copy-on-write by many sequences: "Paged Attention",
 * aidolsgroup.com, section "Example"; agentechip.com "Shared Prefix
 * Caching").  The result equals pa_decode_attention with, for sequence s,
 * block table prefix_blocks ++ suffix_tables[s] and context length
 * prefix_len + suffix_lens[s].  The prefix is attended once per KV head for
 * all S*G query rows together on the tensor cores (each prefix K/V tile read
 * once per 256 query rows), the suffixes by the decode kernel, and one merge
 * combines the partial results.
 *
 * Streams: the prefix kernel runs on a side stream of the library's (one per
 * device, created on first use, highest priority), forked from `stream` by
 * an event and joined back to it before the merge, so that the suffixes'
 * planner and decode on `stream` may run at the same time.  All the call's
 * work follows what was queued on `stream` before it and precedes what is
 * queued after it; the side stream also orders the prefix kernels of calls
 * on different streams.  With PA_PREFIX_SERIAL=1 in the environment every
 * kernel runs on `stream`, one after the other.
 *
 *   prefix_blocks  device int32 [prefix_len / block_size]
 *   prefix_len     tokens; a multiple of block_size and of 16 (0: plain call)
 *   suffix_tables  device int32 rows of max_suffix_blocks valid entries,
 *                  suffix_table_stride elements apart (>= max_suffix_blocks)
 *   suffix_lens    device int32 [S], each <= max_suffix_blocks*block_size
 *   workspace      pa_shared_prefix_workspace_size() bytes, caller-owned
 * Other arguments as for pa_decode_attention.  f16/bf16 caches only
 * (PA_ERR_UNSUPPORTED otherwise). */
pa_status pa_decode_attention_shared_prefix(const void* q, const void* k_cache, const void* v_cache,
                                            int32_t num_blocks, const int32_t* prefix_blocks,
                                            int32_t prefix_len, const int32_t* suffix_tables,
                                            int32_t suffix_table_stride, int32_t max_suffix_blocks,
                                            const int32_t* suffix_lens, int32_t num_seqs,
                                            int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                            int32_t block_size, float scale, int32_t partition_size,
                                            void* workspace, size_t workspace_bytes, void* out,
                                            pa_dtype dtype, void* stream);

/* Largest workspace pa_decode_attention_static can use: 32 MiB. */
#define PA_STATIC_WORKSPACE_BYTES (32u * 1024u * 1024u)

/* pa_decode_attention for callers that cannot allocate device memory.  The
 * pages have no counterpart to this call; it exists for the library's users.
 *
 * Some callers cannot call cudaMalloc: a host framework that has already
 * handed the whole GPU to its own allocator (so a fresh allocation would fail
 * or fragment that pool), or code on a path where cudaMalloc's implicit
 * device-wide synchronisation is not acceptable.  Such callers still own q,
 * the caches, tables, lengths and out, but pass no workspace: the partials of
 * the split-context path live in a static device array of
 * PA_STATIC_WORKSPACE_BYTES that every GPU loading this library holds until
 * the process exits.  This call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).
 *
 * Arguments and results are those of pa_decode_attention without
 * `workspace`/`workspace_bytes`.  PA_ERR_INVALID, with a message naming the
 * size, when pa_decode_workspace_size(...) for these sizes exceeds
 * PA_STATIC_WORKSPACE_BYTES.  That limit applies to partition_size == 0 as
 * well: the single-pass path keeps its work list in the array too (256 bytes
 * plus 16 bytes per sequence and query head).
 *
 * Every call looks up the array's device address in the current device's
 * context (cudaGetSymbolAddress; no allocation).  The first call in a context
 * also loads the library's device code there, so make that first call on a
 * device before any stream capture.  All calls on a device share the one
 * array, which keeps whatever the last call left in it (nothing in it has to
 * start at zero: the work counter is reset and every partial is written
 * before it is read within a call).  Calls issued one after another on one
 * stream are ordered on the array.  Calls that overlap on the GPU -- on
 * different streams, or from different host threads -- race on it; serialise
 * them. */
pa_status pa_decode_attention_static(const void* q, const void* k_cache, const void* v_cache,
                                     int32_t num_blocks, const int32_t* block_tables,
                                     int32_t max_blocks_per_seq, const int32_t* context_lens,
                                     int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                     int32_t head_dim, int32_t block_size, float scale,
                                     int32_t partition_size, void* out, pa_dtype dtype, void* stream);

/* Practical read-bandwidth ceiling (a measurement aid, not a step of the
 * path): read every byte of `buf` (device, 16-byte aligned, `bytes` a
 * multiple of 16) once with streaming 16-byte loads on a grid of 4 CTAs of
 * 512 threads per SM, and XOR-fold what was read into *sink (device uint32).
 * Timing it on a buffer larger than L2 gives the bandwidth a read-only
 * stream such as decode attention can reach on this GPU. */
pa_status pa_read_stream(const void* buf, size_t bytes, uint32_t* sink, void* stream);

/* ---- Step executor ------------------------------------------------------
 * One whole decode step of a batch, host buffers in and out, issued by one
 * call: the slot reservation of pa_reserve_slots on the host, then on the
 * GPU the table/length update (pa_update_block_tables), the copy-on-write
 * copies (pa_copy_blocks), the append (pa_append_kv) and the attention
 * (pa_decode_attention), with the host<->device copies around them
 * (agentechip.com "Implementing a Simplified Paged KV Cache" and "Shared
 * Prefix Caching"; krapton.com "How Paged Attention Works", steps 3-4).
 *
 * Copies run on two streams of the engine's own (upload, download) and the
 * kernels on the caller's `stream`; the engine keeps two device slots for
 * q, k_new, v_new, out and the step's metadata, so step i+1's upload and step
 * i-1's download overlap step i's kernels.  Not thread-safe: one host thread
 * drives an engine. */
typedef struct pa_engine pa_engine;

/* Create an engine for a batch of num_seqs sequences of one layer's cache.
 * host_tables (int32 [num_seqs][max_blocks_per_seq]) and host_lens (int32
 * [num_seqs]) are the caller's host block tables and lengths, and
 * device_tables / device_lens the caller's device copies of them.  Each must
 * already agree with the other before the first step (upload them once).
 * k_cache / v_cache hold pool->num_blocks blocks of pool->block_size rows of
 * [num_kv_heads][head_dim] elements of `dtype`.  All of them stay owned by
 * the caller and must outlive the engine.  partition_size is passed to
 * pa_decode_attention on every step (0 = single pass).  The engine allocates
 * its staging (two slots of q, out, k_new, v_new and metadata, 32 bytes per
 * sequence), the decode workspace, two streams and six events on the current
 * device.  Errors: PA_ERR_INVALID for a bad argument (checked before anything
 * is allocated), PA_ERR_CUDA when an allocation fails. */
pa_status pa_engine_create(pa_pool* pool, int32_t* host_tables, int32_t* host_lens, int32_t num_seqs,
                           int32_t max_blocks_per_seq, int32_t* device_tables, int32_t* device_lens,
                           void* k_cache, void* v_cache, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, pa_dtype dtype, int32_t partition_size, void* stream,
                           pa_engine** engine_out);

/* Wait for everything the engine issued, then free what it allocated. */
void pa_engine_destroy(pa_engine* engine);

/* One decode step for rows [row0, row0 + num_rows) of the batch.
 *   q      host [num_rows][num_q_heads][head_dim]   query of each row
 *   k_new  host [num_rows][num_kv_heads][head_dim]  the new token's K
 *   v_new  host [num_rows][num_kv_heads][head_dim]  the new token's V
 *   out    host [num_rows][num_q_heads][head_dim]   attention output
 * all of `dtype`, page-locked for the copies to overlap (pageable memory
 * works, with copies that block the host).  The call reserves the slots
 * (host tables and lengths change in place), enqueues the copies and kernels
 * and returns without waiting for them.  The caller must leave q, k_new and
 * v_new unchanged, and not read `out`, until the step is done: after the
 * engine's next-but-one step returns, or after pa_engine_synchronize.  The
 * new token attends to itself (it is appended before the attention).
 * slots_out (host int64 [num_rows]) and pairs_out (host int32
 * [num_rows][2]) receive the slot mapping and the copy-on-write pairs when
 * non-NULL; num_pairs_out the number of pairs.  Errors: PA_ERR_INVALID for
 * bad rows, buffers, scale or device; PA_ERR_EXHAUSTED when the pool runs
 * dry (the pool, tables and lengths are then unchanged and nothing is
 * enqueued); PA_ERR_CUDA when a copy or launch fails (the host reservation
 * has then happened but the device state is undefined: destroy the engine
 * and upload the tables again). */
pa_status pa_engine_step(pa_engine* engine, int32_t row0, int32_t num_rows, const void* q,
                         const void* k_new, const void* v_new, void* out, float scale,
                         int64_t* slots_out, int32_t* pairs_out, int32_t* num_pairs_out);

/* Make the caller's stream wait (on the device) for every copy the engine
 * issued; the host does not block. */
pa_status pa_engine_join(pa_engine* engine);

/* Block the host until every step issued so far is done and its output is in
 * host memory. */
pa_status pa_engine_synchronize(pa_engine* engine);

/* Read (and, if reset != 0, clear) the device error word of the current
 * device: 0 = none; 1 = block id outside the pool in a table; 2 =
 * context length beyond the table; 3 = append slot outside the cache; 4 =
 * copy pair id outside the pool; 5 = a pipeline wait of a kernel ran out of
 * time (that kernel returned early and its output is undefined).
 * Synchronous: waits for the device. */
pa_status pa_device_error(int32_t* code_out, int32_t reset);

/* Test hook for the bounded waits of the decode kernel; not a step of the
 * path, and off unless a test turns it on.  Every wait inside the kernels is
 * bounded in time: a wait that runs out sets device error 5, tells the other
 * warps of its CTA to stop, lets the copies already in flight land, and
 * returns, so a lost arrival can never hang the GPU.  With wait_limit_ns > 0
 * (between 1e3 and 2e9) every following pa_decode_attention launch (until
 * the hook is turned off with 0) uses that bound instead of the normal 2 s,
 * and the producer warp of every decode CTA withholds its first pipeline
 * stage, so the consumer's wait for it is certain to run out: the call
 * completes, its output is undefined, and pa_device_error reports 5.
 * Process-wide setting; PA_ERR_INVALID for a bound outside the range. */
pa_status pa_debug_decode_stall(int64_t wait_limit_ns);

/* Which kernel the last pa_decode_attention_shared_prefix call of this
 * thread launched for the prefix: 1 = the SM-pair tensor-core kernel (two-CTA
 * clusters, head_dim 128), 2 = the one-SM tensor-core kernel, 3 = the
 * mma.sync kernel, 0 = none yet.  The SM-pair kernel is the default (it
 * falls back to the one-SM kernel for head_dim 64 or when no cluster of two
 * is resident); PA_PREFIX_PATH=umma in the environment picks the one-SM
 * kernel and PA_PREFIX_PATH=mma the mma.sync kernel.  A test and
 * measurement aid: returns the value, never fails. */
int pa_debug_last_prefix_kernel(void);

/* Message of the last failing call on this thread ("" if none). */
const char* pa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_PA_H */
