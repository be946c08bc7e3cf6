"""Oracle paged decode attention in fp64 (test infrastructure only).

Paging changes where K and V live, not what attention computes: the pages say
the attention kernel follows the block table, loads the blocks and attends
over the keys and values as if they were one concatenated sequence
("PagedAttention Explained: Managing KV Cache Efficiently", section "Block
Tables and Non-Contiguous Storage"), and that paging leaves the model's
computation unchanged (krapton.com, "FAQ": "Does Paged Attention affect model
accuracy?").  So the oracle is that definition written out:

1. gather the sequence's blocks, in logical order, into contiguous
   ``K, V`` of shape ``[length, num_kv_heads, head_dim]`` (the gather of the
   toy cache in "Implementing a Simplified Paged KV Cache");
2. for every query head ``h`` take KV head ``h // (Hq // Hkv)`` (consecutive
   grouping; the pages do not mention grouped-query attention, this is the
   plain reading and reduces to one KV head per query head when Hq == Hkv);
3. ``out = softmax(q . K^T * scale) V`` in float64, one query per
   (sequence, head), over tokens ``0 .. length-1`` with no mask (a single
   decode query is the last position, so every cached token is visible).

A sequence of length 0 yields a zero row (the pages say nothing; this is the
reading used throughout this project).
"""

import numpy as np


def gather_kv(k_cache, v_cache, table, length, block_size):
    """Concatenate the sequence's blocks in table order; keep the first ``length`` rows."""
    length = int(length)
    nblocks = -(-length // block_size)
    ids = [int(b) for b in table[:nblocks]]
    if nblocks == 0:
        shape = (0,) + tuple(k_cache.shape[2:])
        return np.zeros(shape, np.float64), np.zeros(shape, np.float64)
    k = np.concatenate([np.asarray(k_cache[b], np.float64) for b in ids], axis=0)[:length]
    v = np.concatenate([np.asarray(v_cache[b], np.float64) for b in ids], axis=0)[:length]
    return k, v


def oracle_decode_one(q_vec, keys, values, scale):
    """softmax(q . keys^T * scale) . values for one head, all in float64.

    ``q_vec``: [D]; ``keys``, ``values``: [n, D].  The maximum score is
    subtracted before exponentiating (it cancels in the ratio).
    """
    q_vec = np.asarray(q_vec, np.float64)
    keys = np.asarray(keys, np.float64)
    values = np.asarray(values, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1], np.float64)
    scores = (keys @ q_vec) * float(scale)
    weights = np.exp(scores - scores.max())
    return (weights @ values) / weights.sum()


def oracle_decode(q, k_cache, v_cache, block_tables, context_lens, scale, seqs=None, heads=None):
    """Decode attention for every (sequence, query head), float64 result.

    ``q``: [S, Hq, D]; caches: [NB, bs, Hkv, D]; ``block_tables``: [S, MB]
    (or a list of per-sequence lists); ``context_lens``: [S].  ``seqs`` /
    ``heads`` restrict the work to a subset (the rest of the result stays 0),
    for sampled checks at large sizes.
    """
    num_seqs, num_q_heads, head_dim = q.shape
    block_size, num_kv_heads = k_cache.shape[1], k_cache.shape[2]
    if num_q_heads % num_kv_heads != 0:
        raise ValueError("query heads must be a multiple of KV heads")
    group = num_q_heads // num_kv_heads
    out = np.zeros((num_seqs, num_q_heads, head_dim), np.float64)
    seqs = range(num_seqs) if seqs is None else seqs
    heads = range(num_q_heads) if heads is None else heads
    for s in seqs:
        keys, values = gather_kv(k_cache, v_cache, block_tables[s], context_lens[s], block_size)
        for h in heads:
            kv = h // group
            out[s, h] = oracle_decode_one(q[s, h], keys[:, kv, :], values[:, kv, :], scale)
    return out
