"""Prefix caching end to end on the GPU: prompts get their blocks from the
library's content-keyed cache, only uncached tokens are written, and decode
attention equals the oracle over private (unshared) copies of every prompt."""

import math

import numpy as np
import pytest
import torch

from oracle import oracle_decode
from gpu_cases import assert_close
from paged_kv_cache_341_b200 import workloads

pytestmark = pytest.mark.gpu


def test_cached_prompts_attend_like_private_copies():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(41)
    bs, hkv, hq, d = 16, 2, 8, 128
    systems = [list(rng.integers(0, 32000, size=n)) for n in (48, 100, 0, 35)]
    prompts, sys_of = [], []
    for s in range(14):
        k = int(rng.integers(0, len(systems)))
        prompts.append(systems[k] + list(rng.integers(0, 32000, size=int(rng.integers(1, 40)))))
        sys_of.append(k)
    # K/V of a token depend on what precedes it: rows for system tokens come from the
    # system prompt's own values, suffix rows are private to the sequence
    sys_k = [workloads.randn((len(p), hkv, d), "bf16", 100 + i) for i, p in enumerate(systems)]
    sys_v = [workloads.randn((len(p), hkv, d), "bf16", 200 + i) for i, p in enumerate(systems)]
    seq_k, seq_v = [], []
    for s, p in enumerate(prompts):
        n_sys = len(systems[sys_of[s]])
        suf_k = workloads.randn((len(p) - n_sys, hkv, d), "bf16", 300 + s)
        suf_v = workloads.randn((len(p) - n_sys, hkv, d), "bf16", 400 + s)
        seq_k.append(torch.cat([sys_k[sys_of[s]], suf_k]))
        seq_v.append(torch.cat([sys_v[sys_of[s]], suf_v]))
    nb, mb = 200, 16
    cache = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, len(prompts), mb, fill=float("nan"))
    cache.pool.pa_pool_enable_prefix_cache()
    written = 0
    for s, p in enumerate(prompts):
        row = np.full(mb, -1, np.int32)
        cached = cache.pool.pa_seq_alloc_prompt(p, row)
        assert cached % bs == 0 and cached <= len(systems[sys_of[s]])
        cache.tables[s] = row
        cache.lens[s] = len(p)
        j = np.arange(cached, len(p))
        slots = torch.from_numpy((row[j // bs].astype(np.int64) * bs + j % bs)).cuda()
        cache.append(seq_k[s][cached:].cuda(), seq_v[s][cached:].cuda(), slots)
        written += len(p) - cached
    assert written < sum(len(p) for p in prompts)          # some tokens were served from the cache
    cache.upload_tables()
    q_host = workloads.randn((len(prompts), hq, d), "bf16", 7)
    out = torch.empty((len(prompts), hq, d), dtype=torch.bfloat16, device="cuda")
    cache.attend(q_host.cuda(), out, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    # oracle: every prompt in private, contiguous blocks
    kp = np.zeros((len(prompts) * mb, bs, hkv, d))
    vp = np.zeros_like(kp)
    tables = []
    for s, p in enumerate(prompts):
        n = len(p)
        blocks = list(range(s * mb, s * mb + -(-n // bs)))
        for j in range(n):
            kp[blocks[j // bs], j % bs] = seq_k[s][j].double().numpy()
            vp[blocks[j // bs], j % bs] = seq_v[s][j].double().numpy()
        tables.append(blocks)
    ref = oracle_decode(q_host.double().numpy(), kp, vp, tables, [len(p) for p in prompts], 1 / math.sqrt(d))
    assert_close(out.float().cpu().numpy(), ref, "bf16", "prefix-cached prompts")
