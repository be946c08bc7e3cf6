// Host block pool of libpagedattn.so: first-in first-out free list,
// reference counts, sharing and the per-token slot reservation with
// copy-on-write.  Semantics are those declared in include/pa.h; the pages'
// description is in "PagedAttention Explained: Managing KV Cache Efficiently"
// (agentechip.com), sections "Implementing a Simplified Paged KV Cache" and
// "Shared Prefix Caching".
//
// Design: the free list is a ring buffer of num_blocks int32 entries (a block
// is either referenced or queued, never both, so the ring never overflows);
// allocation pops the head, release pushes at the tail.  Every call validates
// first and mutates after, so a failure leaves the pool unchanged.

#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "pa.h"
#include "pa_common.h"

#include "pool_internal.h"

extern "C" {

pa_status pa_pool_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                         pa_pool** out) {
  if (!out) return pa::fail(PA_ERR_INVALID, "pa_pool_create: out is NULL");
  *out = nullptr;
  if (num_blocks < 0 || block_size <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_pool_create: need num_blocks >= 0 and block_size > 0");
  pa_pool* p = new (std::nothrow) pa_pool();
  if (!p) return pa::fail(PA_ERR_INVALID, "pa_pool_create: out of host memory");
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->ring.resize(num_blocks);
  p->refcount.assign(num_blocks, 0);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete p;
        return pa::fail(PA_ERR_INVALID, "pa_pool_create: initial_free_order is not a permutation");
      }
      seen[b] = 1;
      p->ring[i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) p->ring[i] = i;
  }
  p->head = 0;
  p->count = num_blocks;
  *out = p;
  return pa::ok();
}

void pa_pool_destroy(pa_pool* pool) { delete pool; }

pa_status pa_pool_alloc(pa_pool* pool, int32_t n, int32_t* out_ids) {
  if (!pool || n < 0 || (n > 0 && !out_ids)) return pa::fail(PA_ERR_INVALID, "pa_pool_alloc: bad argument");
  if (n > pool->count)
    return pa::fail(PA_ERR_EXHAUSTED, "KV cache exhausted: " + std::to_string(n) + " blocks requested, " +
                                          std::to_string(pool->count) + " free");
  for (int32_t i = 0; i < n; ++i) {
    int32_t b = pool->pop_front();
    pool->refcount[b] = 1;
    out_ids[i] = b;
  }
  return pa::ok();
}

pa_status pa_pool_free(pa_pool* pool, const int32_t* ids, int32_t n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return pa::fail(PA_ERR_INVALID, "pa_pool_free: bad argument");
  // Validate against a scratch count so duplicates are accounted for.
  std::vector<int32_t> want;
  for (int32_t i = 0; i < n; ++i)
    if (!pool->valid_id(ids[i])) return pa::fail(PA_ERR_INVALID, "pa_pool_free: block id out of range");
  if (n > 0) {
    want.assign(pool->num_blocks, 0);
    for (int32_t i = 0; i < n; ++i)
      if (++want[ids[i]] > pool->refcount[ids[i]])
        return pa::fail(PA_ERR_REFCOUNT, "pa_pool_free: block " + std::to_string(ids[i]) +
                                             " released more often than referenced");
  }
  for (int32_t i = 0; i < n; ++i)
    if (--pool->refcount[ids[i]] == 0) {
      pool->forget_hash(ids[i]);
      pool->push_back(ids[i]);
    }
  return pa::ok();
}

pa_status pa_pool_fork(pa_pool* pool, const int32_t* ids, int32_t n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return pa::fail(PA_ERR_INVALID, "pa_pool_fork: bad argument");
  for (int32_t i = 0; i < n; ++i) {
    if (!pool->valid_id(ids[i])) return pa::fail(PA_ERR_INVALID, "pa_pool_fork: block id out of range");
    if (pool->refcount[ids[i]] < 1)
      return pa::fail(PA_ERR_REFCOUNT, "pa_pool_fork: block " + std::to_string(ids[i]) + " is free");
  }
  for (int32_t i = 0; i < n; ++i) ++pool->refcount[ids[i]];
  return pa::ok();
}

pa_status pa_pool_refcount(const pa_pool* pool, int32_t id, int32_t* out) {
  if (!pool || !out || !pool->valid_id(id)) return pa::fail(PA_ERR_INVALID, "pa_pool_refcount: bad argument");
  *out = pool->refcount[id];
  return pa::ok();
}

pa_status pa_pool_num_free(const pa_pool* pool, int32_t* out) {
  if (!pool || !out) return pa::fail(PA_ERR_INVALID, "pa_pool_num_free: bad argument");
  *out = pool->count;
  return pa::ok();
}

pa_status pa_pool_export(const pa_pool* pool, int32_t* refcounts, int32_t* free_list, int32_t* n_free) {
  if (!pool || !n_free) return pa::fail(PA_ERR_INVALID, "pa_pool_export: bad argument");
  if (refcounts) std::memcpy(refcounts, pool->refcount.data(), sizeof(int32_t) * pool->num_blocks);
  if (free_list) {
    int32_t idx = pool->head;
    for (int32_t i = 0; i < pool->count; ++i) {
      free_list[i] = pool->ring[idx];
      idx = (idx + 1 == pool->num_blocks) ? 0 : idx + 1;
    }
  }
  *n_free = pool->count;
  return pa::ok();
}

}  // extern "C"

namespace {

// One reservation; on success reports what changed so a batch can roll back.
struct Undo {
  int32_t logical = -1;      // table entry written
  int32_t prev_entry = -1;   // its previous content
  int32_t taken = -1;        // block popped from the free list, -1 if none
  bool cow = false;          // prev_entry lost a reference (copy-on-write)
};

pa_status reserve_one(pa_pool* pool, int32_t* table, int32_t cap, int32_t* len, int64_t* slot,
                      int32_t* src, int32_t* dst, Undo* undo) {
  const int32_t bs = pool->block_size;
  const int32_t n = *len;
  if (n < 0) return pa::fail(PA_ERR_INVALID, "pa_seq_reserve_slot: negative length");
  const int32_t logical = n / bs;
  const int32_t offset = n % bs;
  if (logical >= cap) return pa::fail(PA_ERR_INVALID, "pa_seq_reserve_slot: block table too small");
  *src = -1;
  *dst = -1;
  if (offset == 0) {
    if (pool->count == 0) return pa::fail(PA_ERR_EXHAUSTED, "KV cache exhausted: no free blocks available");
    int32_t b = pool->pop_front();
    pool->refcount[b] = 1;
    undo->logical = logical;
    undo->prev_entry = table[logical];
    undo->taken = b;
    undo->cow = false;
    table[logical] = b;
  } else {
    int32_t cur = table[logical];
    if (!pool->valid_id(cur) || pool->refcount[cur] < 1)
      return pa::fail(PA_ERR_INVALID, "pa_seq_reserve_slot: table entry is not a live block");
    if (pool->refcount[cur] > 1) {
      if (pool->count == 0)
        return pa::fail(PA_ERR_EXHAUSTED, "KV cache exhausted: no free block for copy-on-write");
      int32_t b = pool->pop_front();
      pool->refcount[b] = 1;
      --pool->refcount[cur];
      undo->logical = logical;
      undo->prev_entry = cur;
      undo->taken = b;
      undo->cow = true;
      table[logical] = b;
      *src = cur;
      *dst = b;
    }
  }
  *slot = static_cast<int64_t>(table[logical]) * bs + offset;
  *len = n + 1;
  return PA_OK;
}

void roll_back(pa_pool* pool, int32_t* table, int32_t* len, const Undo& u) {
  *len -= 1;
  if (u.taken < 0) return;
  pool->refcount[u.taken] = 0;
  pool->unpop_front(u.taken);
  table[u.logical] = u.prev_entry;
  if (u.cow) ++pool->refcount[u.prev_entry];
}

}  // namespace

extern "C" {

pa_status pa_seq_reserve_slot(pa_pool* pool, int32_t* table, int32_t table_cap, int32_t* len, int64_t* slot_out,
                              int32_t* cow_src_out, int32_t* cow_dst_out) {
  if (!pool || !table || !len || !slot_out || !cow_src_out || !cow_dst_out || table_cap < 0)
    return pa::fail(PA_ERR_INVALID, "pa_seq_reserve_slot: bad argument");
  Undo u;
  pa_status st = reserve_one(pool, table, table_cap, len, slot_out, cow_src_out, cow_dst_out, &u);
  return st == PA_OK ? pa::ok() : st;
}

pa_status pa_reserve_slots_with_updates(pa_pool* pool, int32_t* tables, int32_t table_cap, int32_t* lens,
                                        int32_t num_seqs, int32_t row0, int64_t* slots_out, int32_t* pairs_out,
                                        int32_t* num_pairs_out, int32_t* updates_out, int32_t* num_updates_out) {
  if (!pool || num_seqs < 0 || table_cap < 0 || !num_pairs_out || row0 < 0 ||
      (num_seqs > 0 && (!tables || !lens || !slots_out || !pairs_out)) || (updates_out && !num_updates_out))
    return pa::fail(PA_ERR_INVALID, "pa_reserve_slots: bad argument");
  std::vector<Undo> undo(num_seqs);
  int32_t npairs = 0, nupd = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    int32_t src, dst;
    int32_t* table = tables + static_cast<int64_t>(s) * table_cap;
    pa_status st = reserve_one(pool, table, table_cap, lens + s, slots_out + s, &src, &dst, &undo[s]);
    if (st != PA_OK) {
      for (int32_t r = s - 1; r >= 0; --r)
        roll_back(pool, tables + static_cast<int64_t>(r) * table_cap, lens + r, undo[r]);
      return st;
    }
    if (src >= 0) {
      pairs_out[2 * npairs] = src;
      pairs_out[2 * npairs + 1] = dst;
      ++npairs;
    }
    // the reservation wrote a table entry exactly when it took a block: a
    // fresh one at offset 0, or the copy of a shared one
    if (updates_out && undo[s].taken >= 0) {
      updates_out[3 * nupd] = row0 + s;
      updates_out[3 * nupd + 1] = undo[s].logical;
      updates_out[3 * nupd + 2] = table[undo[s].logical];
      ++nupd;
    }
  }
  *num_pairs_out = npairs;
  if (num_updates_out) *num_updates_out = nupd;
  return pa::ok();
}

pa_status pa_reserve_slots(pa_pool* pool, int32_t* tables, int32_t table_cap, int32_t* lens, int32_t num_seqs,
                           int64_t* slots_out, int32_t* pairs_out, int32_t* num_pairs_out) {
  return pa_reserve_slots_with_updates(pool, tables, table_cap, lens, num_seqs, 0, slots_out, pairs_out,
                                       num_pairs_out, nullptr, nullptr);
}

}  // extern "C"
