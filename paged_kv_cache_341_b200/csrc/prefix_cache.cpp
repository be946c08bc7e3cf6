// Prefix caching by block content for the host pool ("Paged Attention",
// aidolsgroup.com, section "Why it matters": each KV-cache block is hashed by
// its tokens and by the tokens before it, so requests that share a system
// prompt reuse the same blocks; agentechip.com "Enabling Automatic Prefix
// Caching").
//
// Hash: 64-bit FNV-1a over the little-endian bytes of the int32 token ids from
// the start of the prompt to the end of the block, i.e. the hash of block i is
// FNV-1a(tokens[0 : (i+1) * block_size]); it is computed incrementally, so a
// block's key covers its own tokens and its whole prefix.  Only full blocks are
// registered.  A hit is confirmed by comparing the stored token ids of the
// block; lookups stop at the first miss (a prompt reuses a prefix of blocks).
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "pa.h"
#include "pa_common.h"
#include "pool_internal.h"

namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv1a_tokens(uint64_t h, const int32_t* tokens, int32_t n) {
  for (int32_t i = 0; i < n; ++i) {
    const uint32_t t = static_cast<uint32_t>(tokens[i]);
    for (int byte = 0; byte < 4; ++byte) {
      h ^= (t >> (8 * byte)) & 0xffu;
      h *= kFnvPrime;
    }
  }
  return h;
}

}  // namespace

extern "C" {

pa_status pa_pool_enable_prefix_cache(pa_pool* pool) {
  if (!pool) return pa::fail(PA_ERR_INVALID, "pa_pool_enable_prefix_cache: pool is NULL");
  if (!pool->prefix_cache) {
    pool->prefix_cache = true;
    pool->hash_of.assign(pool->num_blocks, 0);
    pool->registered.assign(pool->num_blocks, 0);
    pool->tokens_of.assign(static_cast<size_t>(pool->num_blocks) * pool->block_size, 0);
  }
  return pa::ok();
}

pa_status pa_prefix_hash(const int32_t* tokens, int32_t num_tokens, uint64_t seed, uint64_t* out) {
  if (!out || num_tokens < 0 || (num_tokens > 0 && !tokens)) return pa::fail(PA_ERR_INVALID, "pa_prefix_hash: bad argument");
  *out = fnv1a_tokens(seed == 0 ? kFnvOffset : seed, tokens, num_tokens);
  return pa::ok();
}

pa_status pa_seq_alloc_prompt(pa_pool* pool, const int32_t* tokens, int32_t num_tokens, int32_t* table,
                              int32_t table_cap, int32_t* num_cached_tokens) {
  if (!pool || !table || !num_cached_tokens || num_tokens < 0 || (num_tokens > 0 && !tokens))
    return pa::fail(PA_ERR_INVALID, "pa_seq_alloc_prompt: bad argument");
  if (!pool->prefix_cache) return pa::fail(PA_ERR_INVALID, "pa_seq_alloc_prompt: prefix cache not enabled");
  const int32_t bs = pool->block_size;
  const int32_t nblocks = (num_tokens + bs - 1) / bs;
  const int32_t nfull = num_tokens / bs;
  if (nblocks > table_cap) return pa::fail(PA_ERR_INVALID, "pa_seq_alloc_prompt: block table too small");

  // 1) leading full blocks found in the cache (confirmed token by token)
  uint64_t h = kFnvOffset;
  std::vector<uint64_t> hashes(nfull);
  int32_t hits = 0;
  bool searching = true;
  for (int32_t i = 0; i < nfull; ++i) {
    h = fnv1a_tokens(h, tokens + static_cast<size_t>(i) * bs, bs);
    hashes[i] = h;
    if (searching) {
      auto it = pool->by_hash.find(h);
      if (it != pool->by_hash.end() &&
          std::memcmp(&pool->tokens_of[static_cast<size_t>(it->second) * bs], tokens + static_cast<size_t>(i) * bs,
                      sizeof(int32_t) * bs) == 0) {
        table[i] = it->second;
        ++hits;
      } else {
        searching = false;
      }
    }
  }
  // 2) fresh blocks for the rest, all or nothing
  const int32_t fresh = nblocks - hits;
  if (fresh > pool->count)
    return pa::fail(PA_ERR_EXHAUSTED, "KV cache exhausted: " + std::to_string(fresh) + " blocks requested, " +
                                          std::to_string(pool->count) + " free");
  for (int32_t i = 0; i < hits; ++i) ++pool->refcount[table[i]];
  for (int32_t i = hits; i < nblocks; ++i) {
    const int32_t b = pool->pop_front();
    pool->refcount[b] = 1;
    table[i] = b;
    if (i < nfull) {
      // register the new full block (first writer of this content wins)
      if (pool->by_hash.find(hashes[i]) == pool->by_hash.end()) {
        pool->by_hash.emplace(hashes[i], b);
        pool->hash_of[b] = hashes[i];
        pool->registered[b] = 1;
        std::memcpy(&pool->tokens_of[static_cast<size_t>(b) * bs], tokens + static_cast<size_t>(i) * bs,
                    sizeof(int32_t) * bs);
      }
    }
  }
  *num_cached_tokens = hits * bs;
  return pa::ok();
}

pa_status pa_pool_cached_blocks(const pa_pool* pool, int32_t* out) {
  if (!pool || !out) return pa::fail(PA_ERR_INVALID, "pa_pool_cached_blocks: bad argument");
  *out = static_cast<int32_t>(pool->by_hash.size());
  return pa::ok();
}

}  // extern "C"
