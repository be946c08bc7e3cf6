"""Seeded synthetic inputs for the paged decode path.

This module only draws random numbers and states workload shapes.  It does
none of the method's arithmetic (no block tables, no slot arithmetic, no
attention): the library's allocator and the oracle's allocator each turn the
lengths and the pool order drawn here into block tables on their own.

Values: q, K, V ~ N(0, 1) drawn in float32 with torch's CPU generator and
rounded to the cache dtype.  Lengths and pool orders come from
``numpy.random.default_rng(seed)`` with ``seed = 3410 + workload index``.

The five workloads (shapes named after the models whose attention layer they
copy; no weights are involved):

tiny_fp32       4 seqs, lengths {1,16,17,45}, 2 query / 2 KV heads, head_dim 64,
                block 16, pool of 16 blocks in a seeded random order, fp32
llama2_7b_mha   64 seqs, lengths uniform in [128, 4096], 32/32 heads, head_dim
                128, block 16, shuffled pool of 20,000 blocks, fp16
llama3_8b_gqa   256 seqs, lengths log-normal (median 1024, sigma 1 in log
                space) clipped to [16, 8192], 32/8 heads, head_dim 128, block
                16, shuffled pool of 1.1x the blocks needed, bf16
shared_prefix   200 seqs sharing one 30,720-token prefix (1,920 blocks) plus a
                private suffix uniform in [1, 512], 32/8 heads, head_dim 128,
                block 16, bf16
long_70b_gqa    8 seqs, lengths uniform in [16384, 32768], 64/8 heads,
                head_dim 128, block 32, split into 512-token partitions, bf16
"""

import dataclasses
import math

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass
class Workload:
    name: str
    index: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    partition_size: int = 0          # 0 = one pass over the whole context
    num_blocks: int = 0              # filled by lengths()
    max_blocks_per_seq: int = 0      # filled by lengths()
    shared_prefix: int = 0           # tokens shared by every sequence
    append_headroom: int = 128       # tokens each sequence may still grow by

    @property
    def seed(self):
        return 3410 + self.index

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def elem_bytes(self):
        return torch.empty((), dtype=self.torch_dtype).element_size()


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 4, 2, 2, 64, 16, "f32"),
    # partition sizes: the 70B-shaped workload states 512; for the Llama shapes, which state
    # none, 1,024 was the fastest of 256/512/1,024/2,048 on B200
    "llama2_7b_mha": Workload("llama2_7b_mha", 2, 64, 32, 32, 128, 16, "f16", partition_size=1024),
    "llama3_8b_gqa": Workload("llama3_8b_gqa", 3, 256, 32, 8, 128, 16, "bf16", partition_size=1024),
    "shared_prefix": Workload("shared_prefix", 4, 200, 32, 8, 128, 16, "bf16", partition_size=512,
                              shared_prefix=30720),
    "long_70b_gqa": Workload("long_70b_gqa", 5, 8, 64, 8, 128, 32, "bf16", partition_size=512),
}


def get(name, block_size=None):
    """A copy of workload ``name``; ``block_size`` overrides its block size (block-size sweeps)."""
    w = dataclasses.replace(WORKLOADS[name])
    if block_size is not None:
        w.block_size = int(block_size)
    return w


def lengths(w):
    """Context lengths (suffix lengths for ``shared_prefix``), pool size and table width.

    Returns ``lens`` (numpy int64 [S]) and sets ``w.num_blocks`` and
    ``w.max_blocks_per_seq``.  Pool sizes follow the workload recipes: fixed
    16 / 20,000 blocks, otherwise 1.1x the blocks the lengths need (plus one
    private block per sequence for ``shared_prefix`` forks).
    """
    rng = np.random.default_rng(w.seed)
    bs = w.block_size
    if w.name == "tiny_fp32":
        lens = np.array([1, 16, 17, 45], np.int64)
        w.num_blocks = 16
        w.max_blocks_per_seq = 4
    elif w.name == "llama2_7b_mha":
        lens = rng.integers(128, 4096, size=w.num_seqs, endpoint=True).astype(np.int64)
        w.num_blocks = 20000
        w.max_blocks_per_seq = -(-(4096 + w.append_headroom) // bs)
    elif w.name == "llama3_8b_gqa":
        raw = rng.lognormal(mean=math.log(1024.0), sigma=1.0, size=w.num_seqs)
        lens = np.clip(np.floor(raw), 16, 8192).astype(np.int64)
        need = int(sum(-(-int(n) // bs) for n in lens))
        w.num_blocks = int(math.ceil(1.1 * need))
        w.max_blocks_per_seq = -(-(8192 + w.append_headroom) // bs)
    elif w.name == "shared_prefix":
        lens = rng.integers(1, 512, size=w.num_seqs, endpoint=True).astype(np.int64)
        prefix_blocks = w.shared_prefix // bs
        need = prefix_blocks + int(sum(-(-int(n) // bs) for n in lens)) + 2 * w.num_seqs
        w.num_blocks = int(math.ceil(1.1 * need))
        w.max_blocks_per_seq = -(-(w.shared_prefix + 512 + w.append_headroom) // bs)
    elif w.name == "long_70b_gqa":
        lens = rng.integers(16384, 32768, size=w.num_seqs, endpoint=True).astype(np.int64)
        need = int(sum(-(-int(n) // bs) for n in lens))
        w.num_blocks = int(math.ceil(1.1 * need))
        w.max_blocks_per_seq = -(-(32768 + w.append_headroom) // bs)
    else:
        raise KeyError(w.name)
    return lens


def pool_order(num_blocks, seed):
    """Seeded starting order of the free list (a permutation of 0..N-1)."""
    return np.random.default_rng(seed + 7919).permutation(num_blocks).astype(np.int32)


def randn(shape, dtype, seed):
    """N(0,1) values drawn in float32 on the CPU, rounded to ``dtype`` (torch tensor)."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(DTYPES[dtype] if isinstance(dtype, str) else dtype)


def fill_blocks(w, block_ids, seed, poison_unused=False):
    """K and V pools ``[num_blocks, block_size, Hkv, D]`` with N(0,1) values in ``block_ids``.

    Blocks are filled in the order given (K for all of them, then V); blocks
    not listed hold 0, or NaN when ``poison_unused`` (used to show that
    nothing outside a sequence's tokens is ever read).
    """
    shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
    fill = float("nan") if poison_unused else 0.0
    k = torch.full(shape, fill, dtype=w.torch_dtype)
    v = torch.full(shape, fill, dtype=w.torch_dtype)
    ids = torch.as_tensor(np.asarray(block_ids, np.int64))
    if ids.numel():
        sub = (ids.numel(),) + shape[1:]
        k[ids] = randn(sub, w.dtype, seed)
        v[ids] = randn(sub, w.dtype, seed + 1)
    return k, v


def queries(w, seed, num_seqs=None):
    """One decode query per (sequence, query head): ``[S, Hq, D]``."""
    s = w.num_seqs if num_seqs is None else num_seqs
    return randn((s, w.num_q_heads, w.head_dim), w.dtype, seed)


def new_tokens(w, seed, num_tokens):
    """K and V rows for tokens appended this step: two ``[T, Hkv, D]`` tensors."""
    shape = (num_tokens, w.num_kv_heads, w.head_dim)
    return randn(shape, w.dtype, seed), randn(shape, w.dtype, seed + 1)
