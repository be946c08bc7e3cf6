"""pa_decode_attention_static: decode attention for callers that cannot
allocate device memory -- for example a host framework that has already
handed the whole GPU to its own allocator, or a path on which cudaMalloc's
implicit device-wide synchronisation is not allowed.  Its work list and
split-context partials live in a static 32 MiB array inside the library
instead of a caller workspace.

Checked through the C ABI:
* against the oracle, element by element, within the 16-bit tolerance;
* against pa_decode_attention with a caller-allocated workspace on the same
  inputs, bit for bit (the same kernels run in the same configuration);
* on calls in a row with different inputs, both synchronised one by one and
  queued back to back on one stream with no synchronisation between them
  (every call shares the one array, so a call must not be disturbed by what
  the call before it left there, or by that call still running);
* single pass (partition_size 0, which also keeps its work list in the
  array) and split context.

This file is collected last so a failure here never hides another test's
result.
"""

import math

import numpy as np
import pytest
import torch

from oracle import oracle_decode
from gpu_cases import AsF64, TORCH, assert_close, build_pool_contents, full_table_case
from paged_kv_cache_341_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa as mod
    assert mod.pa_device_error(reset=True) == 0
    return mod


def make_case(lens, seed, dtype="bf16", hq=32, hkv=8, d=128, bs=16):
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
    q = workloads.randn((s, hq, d), dtype, seed + 5)
    return cache, q, k, v


def oracle_out(cache, q_host, k, v, lens):
    d = q_host.shape[2]
    return oracle_decode(q_host.double().numpy(), AsF64(k), AsF64(v), [list(r) for r in cache.tables], lens,
                         1.0 / math.sqrt(d))


@pytest.mark.parametrize("partition", [0, 512, 256])
def test_static_matches_oracle_and_caller_workspace_twice_in_a_row(pa, partition):
    rng = np.random.default_rng(2024 + partition)
    first = [int(x) for x in rng.integers(1, 4000, size=24)] + [0, 1, 513, 8000]
    second = [int(x) for x in rng.integers(1, 1500, size=40)] + [700]
    for lens, seed in ((first, 11), (second, 12)):
        cache, q_host, k, v = make_case(lens, seed)
        q = q_host.cuda()
        s, hq, d = q.shape
        scale = 1.0 / math.sqrt(d)
        ws = pa.decode_workspace(s, hq, d, cache.max_blocks, cache.block_size, partition)
        assert ws.numel() <= pa.STATIC_WORKSPACE_BYTES
        ref = torch.full_like(q, float("nan"))
        pa.pa_decode_attention(q, cache.k_cache, cache.v_cache, cache.d_tables, cache.d_lens, scale, ref,
                               partition_size=partition, workspace=ws)
        got = torch.full_like(q, float("nan"))
        pa.pa_decode_attention_static(q, cache.k_cache, cache.v_cache, cache.d_tables, cache.d_lens, scale, got,
                                      partition_size=partition)
        torch.cuda.synchronize()
        assert pa.pa_device_error() == 0
        got_h, ref_h = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.array_equal(got_h, ref_h), "static call differs from the caller-workspace call"
        assert_close(got_h, oracle_out(cache, q_host, k, v, lens), "bf16",
                     "static vs oracle, partition %d, %d sequences" % (partition, len(lens)))


@pytest.mark.parametrize("partition", [0, 512])
def test_static_calls_queued_back_to_back(pa, partition):
    """Four static calls with different queries and lengths, issued with no
    synchronisation in between: each must match the oracle."""
    s, mb, bs, hq, hkv, d = 48, 64, 16, 32, 8, 128
    cache, k, v, tables = full_table_case(s, mb, bs, hkv, d, "bf16", seed=5151)
    rng = np.random.default_rng(5152)
    cap = mb * bs
    lens_sets = [[int(x) for x in rng.integers(cap // 2, cap + 1, size=s)],
                 [int(x) for x in rng.integers(1, 100, size=s)],
                 [int(x) for x in rng.integers(0, cap + 1, size=s)],
                 [cap] * (s // 2) + [1] * (s - s // 2)]
    qs = [workloads.randn((s, hq, d), "bf16", 5160 + i) for i in range(4)]
    d_lens = [torch.tensor(l, dtype=torch.int32, device="cuda") for l in lens_sets]
    d_q = [q.cuda() for q in qs]
    outs = [torch.full((s, hq, d), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    scale = 1.0 / math.sqrt(d)
    torch.cuda.synchronize()
    for i in range(4):
        pa.pa_decode_attention_static(d_q[i], cache.k_cache, cache.v_cache, cache.d_tables, d_lens[i], scale,
                                      outs[i], partition_size=partition)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    kd, vd = AsF64(k), AsF64(v)
    for i in range(4):
        ref = oracle_decode(qs[i].double().numpy(), kd, vd, tables, lens_sets[i], scale)
        assert_close(outs[i].float().cpu().numpy(), ref, "bf16", "queued static call %d, partition %d" % (i, partition))


def test_static_rejects_sizes_beyond_its_array(pa):
    cache, q_host, _, _ = make_case([4000] * 8, 13)
    q = q_host.cuda()
    s, hq, d = q.shape
    need = pa.pa_decode_workspace_size(s, hq, d, 40000, cache.block_size, 16)
    assert need > pa.STATIC_WORKSPACE_BYTES
    big_tables = torch.zeros((s, 40000), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_decode_attention_static(q, cache.k_cache, cache.v_cache, big_tables, cache.d_lens, 0.1, out,
                                      partition_size=16)
    assert e.value.status == pa.PA_ERR_INVALID and "static" in str(e.value)
