// Internal state of the host block pool (shared by pool.cpp and
// prefix_cache.cpp; not part of the C ABI).
#ifndef PAGEDATTN_POOL_INTERNAL_H
#define PAGEDATTN_POOL_INTERNAL_H

#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_pool {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> ring;      // free list storage, capacity num_blocks
  int32_t head = 0;               // index of the front entry
  int32_t count = 0;              // entries queued
  std::vector<int32_t> refcount;  // per block id

  int32_t pop_front() {
    int32_t b = ring[head];
    head = (head + 1 == num_blocks) ? 0 : head + 1;
    --count;
    return b;
  }
  void push_back(int32_t b) {
    int32_t tail = head + count;
    if (tail >= num_blocks) tail -= num_blocks;
    ring[tail] = b;
    ++count;
  }
  // Undo the most recent pop_front (used to roll back multi-step calls).
  void unpop_front(int32_t b) {
    head = (head == 0) ? num_blocks - 1 : head - 1;
    ring[head] = b;
    ++count;
  }
  bool valid_id(int32_t b) const { return b >= 0 && b < num_blocks; }

  // Prefix cache (pa_pool_enable_prefix_cache): chained content hash of every
  // registered full block -> block id, and each registered block's tokens.
  bool prefix_cache = false;
  std::unordered_map<uint64_t, int32_t> by_hash;
  std::vector<uint64_t> hash_of;          // per block id, valid when registered[b]
  std::vector<char> registered;           // per block id
  std::vector<int32_t> tokens_of;         // [num_blocks][block_size] token ids of registered blocks

  // A block that goes back to the free list is no longer findable by hash.
  void forget_hash(int32_t b) {
    if (!prefix_cache || !registered[b]) return;
    auto it = by_hash.find(hash_of[b]);
    if (it != by_hash.end() && it->second == b) by_hash.erase(it);
    registered[b] = 0;
  }
};


#endif
