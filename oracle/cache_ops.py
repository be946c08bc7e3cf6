"""Oracle cache-maintenance operations (test infrastructure only).

Cache layout: one array per K and V of shape ``[num_blocks, block_size,
num_kv_heads, head_dim]`` -- every physical block holds ``block_size`` token
rows of ``(num_kv_heads, head_dim)``, the per-block shape given for the toy
block in "PagedAttention Explained: Managing KV Cache Efficiently",
section "Implementing a Simplified Paged KV Cache".

Both operations move bits only, so they work on any numpy dtype (16-bit
caches may be passed as their uint16 bit patterns).
"""

import numpy as np


def oracle_append(k_cache, v_cache, k_new, v_new, slot_mapping):
    """Write token ``t``'s K/V row into flat slot ``slot_mapping[t]`` (in place).

    A flat slot ``x`` names block ``x // block_size``, row ``x % block_size``
    (the write of a token into its block's next position, agentechip.com
    "Implementing a Simplified Paged KV Cache").  Negative slots mean "no
    write" (padding entries).
    """
    block_size = k_cache.shape[1]
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        block, row = slot // block_size, slot % block_size
        k_cache[block, row] = k_new[t]
        v_cache[block, row] = v_new[t]


def oracle_copy_blocks(k_cache, v_cache, pairs):
    """For each ``(src, dst)`` pair copy the whole block, K and V (in place).

    This is the copy half of copy-on-write for blocks shared by several
    sequences (krapton.com "How Paged Attention Works", step 4; agentechip.com
    "Shared Prefix Caching").  Pairs are applied in order.
    """
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]
