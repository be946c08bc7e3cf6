"""pa_decode_attention_static: decode attention for callers that cannot
allocate device memory (for example a host framework that has already handed
the whole GPU to its own allocator, or a path where cudaMalloc's implicit
synchronisation is not allowed).  Its split-context partials live in a static
32 MiB array inside the library instead of a caller workspace.

Checked through the C ABI against pa_decode_attention with a caller-allocated
workspace, on two calls in a row with different inputs (the second call must
not be disturbed by what the first left in the shared array).  This file is
collected last so a failure here never hides another test's result.
"""

import math

import numpy as np
import pytest
import torch

from gpu_cases import TORCH, assert_close, build_pool_contents
from paged_kv_cache_341_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa as mod
    return mod


def make_case(pa, lens, seed, dtype="bf16", hq=32, hkv=8, d=128, bs=16):
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(seed)
    s = len(lens)
    nb = sum(-(-n // bs) for n in lens) + 4
    mb = max(-(-n // bs) for n in lens) + 1
    cache = PagedKVCache(nb, bs, hkv, d, TORCH[dtype], s, mb, initial_free_order=rng.permutation(nb))
    for row, n in enumerate(lens):
        cache.allocate(row, n)
    k, v = build_pool_contents((nb, bs, hkv, d), dtype, cache.tables, lens, bs, seed)
    cache.k_cache.copy_(k)
    cache.v_cache.copy_(v)
    cache.upload_tables()
    q = workloads.randn((s, hq, d), dtype, seed + 5).cuda()
    return cache, q


def run_both(pa, cache, q, partition):
    s, hq, d = q.shape
    scale = 1.0 / math.sqrt(d)
    ws = pa.decode_workspace(s, hq, d, cache.max_blocks, cache.block_size, partition)
    assert ws is None or ws.numel() <= pa.STATIC_WORKSPACE_BYTES
    ref = torch.empty_like(q)
    pa.pa_decode_attention(q, cache.k_cache, cache.v_cache, cache.d_tables, cache.d_lens, scale, ref,
                           partition_size=partition, workspace=ws)
    got = torch.full_like(q, float("nan"))
    pa.pa_decode_attention_static(q, cache.k_cache, cache.v_cache, cache.d_tables, cache.d_lens, scale, got,
                                  partition_size=partition)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    return got.float().cpu().numpy(), ref.float().cpu().numpy()


def test_static_workspace_matches_caller_workspace_twice_in_a_row(pa):
    rng = np.random.default_rng(2024)
    first = [int(x) for x in rng.integers(1, 4000, size=24)] + [1, 513, 8000]
    second = [int(x) for x in rng.integers(1, 1500, size=40)] + [700]
    for lens, seed, partition in ((first, 11, 512), (second, 12, 256)):
        cache, q = make_case(pa, lens, seed)
        got, ref = run_both(pa, cache, q, partition)
        assert_close(got, ref, "bf16", "static vs caller workspace, partition %d" % partition)


def test_static_rejects_sizes_beyond_its_array(pa):
    cache, q = make_case(pa, [4000] * 8, 13)
    s, hq, d = q.shape
    need = pa.pa_decode_workspace_size(s, hq, d, 40000, cache.block_size, 16)
    assert need > pa.STATIC_WORKSPACE_BYTES
    big_tables = torch.zeros((s, 40000), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_decode_attention_static(q, cache.k_cache, cache.v_cache, big_tables, cache.d_lens, 0.1, out,
                                      partition_size=16)
    assert e.value.status == pa.PA_ERR_INVALID and "static" in str(e.value)
