"""Plain CPU oracle for the paged-KV-cache decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library, its
Python binding) may import, call or link anything here.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` use it.

The oracle is written from the descriptions on four web pages about
PagedAttention and shares no code with the CUDA path:

* "PagedAttention Explained: Managing KV Cache Efficiently" (agentechip.com),
  sections "Block Tables and Non-Contiguous Storage", "Shared Prefix Caching"
  and "Implementing a Simplified Paged KV Cache";
* "Master Paged Attention for LLM Inference: Boost Throughput & Cut Costs"
  (krapton.com), sections "How Paged Attention Works: The Mechanics" and "FAQ";
* "What is PagedAttention" (aitechboss.com), section "How PagedAttention Works",
  steps 1-4;
* "Paged Attention" glossary (aidolsgroup.com), sections "Full definition" and
  "Example".

Modules:

``pool``       host block pool: FIFO free list, refcounts, fork and the
               per-token slot reservation with copy-on-write.
``cache_ops``  the two cache-maintenance operations: write of new K/V into
               slots, and whole-block copy.
``attention``  gather of a sequence's blocks into contiguous K/V and plain
               fp64 softmax(q K^T * scale) V, one query per (sequence, head).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
invariants, a library routine (torch's CPU scaled_dot_product_attention in
fp64) and the worked example printed on the agentechip page.  No function
here is "parity unpinned".
"""

from .pool import OraclePool, PoolExhausted, RefcountError, InvalidRequest, fnv1a64, token_bytes
from .cache_ops import oracle_append, oracle_copy_blocks
from .attention import gather_kv, oracle_decode, oracle_decode_one

__all__ = [
    "OraclePool", "PoolExhausted", "RefcountError", "InvalidRequest", "fnv1a64", "token_bytes",
    "oracle_append", "oracle_copy_blocks",
    "gather_kv", "oracle_decode", "oracle_decode_one",
]
