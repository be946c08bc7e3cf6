"""Oracle host block pool (test infrastructure only; see ``oracle/__init__``).

What it models, from the pages:

* A fixed number of equally sized physical blocks, each holding K and V for
  ``block_size`` tokens, kept in one pool; a sequence reaches its blocks through
  its own block table, which need not be contiguous
  ("PagedAttention Explained: Managing KV Cache Efficiently", section
  "Block Tables and Non-Contiguous Storage"; krapton.com "How Paged Attention
  Works: The Mechanics", steps 1-3).
* Blocks are handed out only when a sequence needs one: a new block is taken
  when a token lands at offset 0 of a block, and the pool running dry is an
  error ("KV cache exhausted") -- agentechip.com, section "Implementing a
  Simplified Paged KV Cache".
* The free list is first-in first-out: allocation takes the front entry,
  release puts a block at the back, and the untouched list starts as
  0..N-1 (same section).  A caller may instead pass a permutation as the
  starting order (used for the "shuffled pool" workloads).
* Each block carries a reference count: 1 on allocation, +1 per sharer,
  -1 per release; at 0 it returns to the free list (same section, and
  "Shared Prefix Caching").
* Blocks shared between sequences are copied before a write
  (krapton.com step 4 "Shared Blocks"; agentechip.com "Shared Prefix
  Caching").  The pages give no rule for *when*; the reading used here is the
  plainest one: appending a token at offset > 0 of a block whose count is
  above 1 first moves the writer onto a fresh block (copy-on-write); a token
  at offset 0 always starts a fresh block, so nothing is copied.
* Every failing call leaves the pool exactly as it was (all or nothing).

Plain Python lists on purpose: slow, but each rule above is one visible line.
"""


FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3


def fnv1a64(data, h=FNV_OFFSET):
    """64-bit FNV-1a of a byte string, continued from ``h``."""
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & 0xFFFFFFFFFFFFFFFF
    return h


def token_bytes(tokens):
    """int32 token ids as little-endian bytes (the key's input)."""
    out = bytearray()
    for t in tokens:
        out += (int(t) & 0xFFFFFFFF).to_bytes(4, "little")
    return bytes(out)


class PoolExhausted(RuntimeError):
    """No free block is left for a request (the pages' "KV cache exhausted")."""


class RefcountError(RuntimeError):
    """A release or share names a block whose count does not allow it."""


class InvalidRequest(ValueError):
    """Out-of-range block id, negative count, or a table too short."""


class OraclePool:
    def __init__(self, num_blocks, block_size, initial_free_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise InvalidRequest("num_blocks must be >= 0 and block_size > 0")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if initial_free_order is None:
            order = list(range(self.num_blocks))
        else:
            order = [int(b) for b in initial_free_order]
            if sorted(order) != list(range(self.num_blocks)):
                raise InvalidRequest("initial_free_order must be a permutation of 0..N-1")
        self.free_list = order
        self.refcounts = [0] * self.num_blocks
        self.prefix_cache = None          # key -> block id, once enabled
        self.block_key = {}               # registered block id -> (key, its token ids)

    # -- pool-level operations ------------------------------------------------

    def _check_id(self, b):
        if not (0 <= b < self.num_blocks):
            raise InvalidRequest("block id %d out of range" % b)

    def num_free(self):
        return len(self.free_list)

    def alloc(self, n):
        """Take ``n`` blocks from the front of the free list, each with count 1."""
        if n < 0:
            raise InvalidRequest("negative allocation")
        if n > len(self.free_list):
            raise PoolExhausted("KV cache exhausted: %d requested, %d free" % (n, len(self.free_list)))
        taken = []
        for _ in range(n):
            b = self.free_list.pop(0)
            self.refcounts[b] = 1
            taken.append(b)
        return taken

    def free(self, ids):
        """Drop one reference per listed id; a block reaching 0 goes to the back."""
        ids = [int(b) for b in ids]
        wanted = {}
        for b in ids:
            self._check_id(b)
            wanted[b] = wanted.get(b, 0) + 1
        for b, k in wanted.items():
            if self.refcounts[b] < k:
                raise RefcountError("block %d has count %d, %d releases asked" % (b, self.refcounts[b], k))
        for b in ids:
            self.refcounts[b] -= 1
            if self.refcounts[b] == 0:
                self._forget(b)
                self.free_list.append(b)

    def fork(self, ids):
        """Add one reference per listed id (a second sequence now shares it)."""
        ids = [int(b) for b in ids]
        for b in ids:
            self._check_id(b)
            if self.refcounts[b] < 1:
                raise RefcountError("cannot share free block %d" % b)
        for b in ids:
            self.refcounts[b] += 1

    # -- prefix caching by block content --------------------------------------
    # "Paged Attention" (aidolsgroup.com), "Why it matters": a block is hashed
    # by its tokens and the tokens before it, so prompts sharing a prefix share
    # its blocks.  Key of full block i: FNV-1a 64 of the bytes of tokens
    # [0, (i+1)*block_size).  Only full blocks are registered; the first block
    # registered under a key keeps it; a block leaves the cache when freed.

    def enable_prefix_cache(self):
        if self.prefix_cache is None:
            self.prefix_cache = {}

    def _forget(self, b):
        if self.prefix_cache is None or b not in self.block_key:
            return
        key, _ = self.block_key.pop(b)
        if self.prefix_cache.get(key) == b:
            del self.prefix_cache[key]

    def alloc_prompt(self, tokens):
        """Table (list of block ids) for a new sequence holding ``tokens``, and
        how many leading tokens sit in blocks found in the cache."""
        if self.prefix_cache is None:
            raise InvalidRequest("prefix cache not enabled")
        bs = self.block_size
        n = len(tokens)
        nblocks = -(-n // bs)
        keys = []
        h = FNV_OFFSET
        for i in range(n // bs):
            # FNV-1a is a byte stream: continuing it over block i's bytes gives the
            # hash of everything up to the end of block i
            h = fnv1a64(token_bytes(tokens[i * bs:(i + 1) * bs]), h)
            keys.append(h)
        table = []
        for i, key in enumerate(keys):
            b = self.prefix_cache.get(key)
            if b is None or self.block_key[b][1] != list(tokens[i * bs:(i + 1) * bs]):
                break
            table.append(b)
        hits = len(table)
        if nblocks - hits > len(self.free_list):
            raise PoolExhausted("KV cache exhausted: %d blocks requested, %d free" % (nblocks - hits,
                                                                                      len(self.free_list)))
        for b in table:
            self.refcounts[b] += 1
        for i in range(hits, nblocks):
            b = self.free_list.pop(0)
            self.refcounts[b] = 1
            table.append(b)
            if i < len(keys) and keys[i] not in self.prefix_cache:
                self.prefix_cache[keys[i]] = b
                self.block_key[b] = (keys[i], list(tokens[i * bs:(i + 1) * bs]))
        return table, hits * bs

    def refcount(self, b):
        self._check_id(b)
        return self.refcounts[b]

    def export(self):
        """Copies of (refcounts per block id, free list front to back)."""
        return list(self.refcounts), list(self.free_list)

    # -- per-sequence slot reservation ----------------------------------------

    def reserve_slot(self, table, length, capacity=None):
        """Reserve the slot for token number ``length`` of one sequence.

        ``table`` is the sequence's block table (a Python list, logical block
        index -> physical id), changed in place.  Returns
        ``(slot, new_length, cow_src, cow_dst)``; ``slot`` is the flat index
        ``physical_block * block_size + offset`` and ``cow_src, cow_dst`` are
        -1 unless a shared block had to be copied before this write.
        """
        bs = self.block_size
        logical = length // bs
        offset = length % bs
        if length < 0:
            raise InvalidRequest("negative length")
        if capacity is not None and logical >= capacity:
            raise InvalidRequest("block table capacity %d too small" % capacity)
        cow_src, cow_dst = -1, -1
        if offset == 0:
            # The token opens a new logical block: take a fresh physical one.
            if len(table) != logical:
                raise InvalidRequest("table holds %d blocks, expected %d" % (len(table), logical))
            if not self.free_list:
                raise PoolExhausted("KV cache exhausted: no free blocks available")
            fresh = self.free_list.pop(0)
            self.refcounts[fresh] = 1
            table.append(fresh)
        else:
            if len(table) != logical + 1:
                raise InvalidRequest("table holds %d blocks, expected %d" % (len(table), logical + 1))
            current = table[logical]
            self._check_id(current)
            if self.refcounts[current] < 1:
                raise InvalidRequest("table names free block %d" % current)
            if self.refcounts[current] > 1:
                # Shared and partly filled: the writer moves to a private copy.
                if not self.free_list:
                    raise PoolExhausted("KV cache exhausted: no free block for copy-on-write")
                fresh = self.free_list.pop(0)
                self.refcounts[fresh] = 1
                self.refcounts[current] -= 1
                table[logical] = fresh
                cow_src, cow_dst = current, fresh
        slot = table[logical] * bs + offset
        return slot, length + 1, cow_src, cow_dst
