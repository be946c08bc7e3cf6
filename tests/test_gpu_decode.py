"""GPU parity of the decode path against the oracle (needs a B200).

Attention: fp32 cache max-abs 1e-5; fp16/bf16 |gpu - ref| <= 2e-2 + 1e-2|ref|.
Append, copy-on-write copy, tables and refcounts: bit-exact.
"""

import math

import numpy as np
import pytest
import torch

from oracle import OraclePool, oracle_append, oracle_copy_blocks, oracle_decode
from gpu_cases import TORCH, AsF64, assert_close, build_pool_contents
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


def run_decode(pa, dtype, hq, hkv, d, bs, lens, partition, seed, q_scale=1.0, scale=None, workspace=True):
    """Build the case through the library pool, run the kernel, return (gpu out, oracle out)."""
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(seed)
    s = len(lens)
    nb = sum(-(-n // bs) for n in lens) + 3
    mb = max(1, max(-(-n // bs) for n in lens)) + 1
    order = rng.permutation(nb).astype(np.int32)
    cache = PagedKVCache(nb, bs, hkv, d, TORCH[dtype], s, mb, initial_free_order=order)
    for row, n in enumerate(lens):
        cache.allocate(row, n)
    k_host, v_host = build_pool_contents((nb, bs, hkv, d), dtype, cache.tables, lens, bs, seed)
    cache.k_cache.copy_(k_host)
    cache.v_cache.copy_(v_host)
    cache.upload_tables()
    q_host = (workloads.randn((s, hq, d), "f32", seed + 2) * q_scale).to(TORCH[dtype])
    q = q_host.cuda()
    out = torch.full((s, hq, d), float("nan"), dtype=TORCH[dtype], device="cuda")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ws = pa.decode_workspace(s, hq, d, mb, bs, partition) if workspace else None
    cache.attend(q, out, scale, partition, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    ref = oracle_decode(q_host.double().numpy(), AsF64(k_host), AsF64(v_host),
                        [list(r) for r in cache.tables], lens, scale)
    return out.float().cpu().numpy(), ref, v_host, cache


LENS = [0, 1, 15, 16, 17, 100, 300]


@pytest.fixture(params=["mma", "alu"])
def path(request, monkeypatch):
    """Consumer of 16-bit caches: tensor cores (default) or CUDA cores."""
    if request.param == "alu":
        monkeypatch.setenv("PA_DECODE_PATH", "alu")
    else:
        monkeypatch.delenv("PA_DECODE_PATH", raising=False)
    return request.param


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 4), (16, 4), (16, 2)])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("partition", [0, 64])
def test_decode_matches_oracle(pa, path, dtype, d, hq, hkv, bs, partition):
    if dtype == "f32" and path == "mma":
        pytest.skip("float32 caches always take the CUDA-core consumer")
    gpu, ref, _, _ = run_decode(pa, dtype, hq, hkv, d, bs, LENS, partition, seed=hq * 7 + hkv + d + bs + partition)
    assert_close(gpu, ref, dtype, "%s dtype=%s d=%d hq=%d hkv=%d bs=%d p=%d" % (path, dtype, d, hq, hkv, bs,
                                                                             partition))


@pytest.mark.parametrize("partition", [0, 512, 16])
def test_many_units_per_cta(pa, path, partition):
    rng = np.random.default_rng(77)
    lens = [int(x) for x in rng.integers(1, 3000, size=300)] + [0, 1, 8192]
    gpu, ref, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, partition, seed=9)
    assert_close(gpu, ref, "bf16", "p=%d" % partition)


def test_round_robin_without_workspace(pa, path):
    """No workspace (single pass only): units dealt round-robin instead of by counter."""
    rng = np.random.default_rng(78)
    lens = [int(x) for x in rng.integers(1, 2500, size=200)] + [0, 1]
    gpu, ref, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 0, seed=10, workspace=False)
    assert_close(gpu, ref, "bf16", "round robin")


@pytest.mark.parametrize("tile_heads", [1, 2, 4])
def test_tile_heads_override(pa, path, monkeypatch, tile_heads):
    monkeypatch.setenv("PA_DECODE_TILE_HEADS", str(tile_heads))
    lens = [3, 16, 600, 1300]
    gpu, ref, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 256, seed=31)
    assert_close(gpu, ref, "bf16", "tile heads %d" % tile_heads)


def test_single_token_returns_value_exactly(pa, path):
    for dtype in ("f32", "bf16", "f16"):
        gpu, ref, v_host, cache = run_decode(pa, dtype, 8, 2, 128, 16, [1, 1, 1], 0, seed=5, q_scale=10.0)
        for s in range(3):
            blk = int(cache.tables[s, 0])
            for h in range(8):
                expect = v_host[blk, 0, h // 4].float().numpy()
                assert np.array_equal(gpu[s, h], expect), (dtype, s, h)
        # split path with one token per sequence too
        gpu2, _, _, _ = run_decode(pa, dtype, 8, 2, 128, 16, [1, 1, 1], 16, seed=5, q_scale=10.0)
        assert np.array_equal(gpu2, gpu)


def test_zero_scale_and_large_scores(pa, path):
    lens = [5, 33, 200]
    gpu, ref, _, _ = run_decode(pa, "f32", 4, 2, 64, 16, lens, 0, seed=11, scale=0.0)
    assert_close(gpu, ref, "f32", "scale=0")
    gpu, ref, _, _ = run_decode(pa, "f32", 4, 2, 64, 16, lens, 32, seed=12, q_scale=30.0)
    assert_close(gpu, ref, "f32", "q x30")
    gpu, ref, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 0, seed=13, q_scale=30.0)
    assert_close(gpu, ref, "bf16", "q x30")


def test_split_matches_single_pass(pa, path):
    lens = [1, 40, 513, 1000, 2048]
    a, ref, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 0, seed=21)
    b, _, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 4096, seed=21)     # one partition each
    assert np.array_equal(a, b)
    c, _, _, _ = run_decode(pa, "bf16", 32, 8, 128, 16, lens, 128, seed=21)
    assert_close(c, ref, "bf16", "p=128")


def test_append_and_copy_bit_exact(pa):
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(3)
    for dtype, hkv, d, bs in (("bf16", 8, 128, 16), ("f32", 2, 64, 16), ("f16", 4, 128, 32)):
        nb, s = 40, 6
        cache = PagedKVCache(nb, bs, hkv, d, TORCH[dtype], s, 8)
        k0 = workloads.randn((nb, bs, hkv, d), dtype, 100)
        v0 = workloads.randn((nb, bs, hkv, d), dtype, 101)
        cache.k_cache.copy_(k0)
        cache.v_cache.copy_(v0)
        slots = rng.choice(nb * bs, size=25, replace=False).astype(np.int64)
        slots[[3, 9]] = -1
        kn = workloads.randn((25, hkv, d), dtype, 102)
        vn = workloads.randn((25, hkv, d), dtype, 103)
        cache.append(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda())
        pairs = np.array([[1, 30], [7, 2], [12, 13]], np.int32)
        cache.copy_blocks(torch.from_numpy(pairs).cuda())
        torch.cuda.synchronize()
        assert pa.pa_device_error() == 0
        # oracle on the raw bits
        bits = torch.int16 if dtype != "f32" else torch.int32
        ko, vo = k0.view(bits).numpy().copy(), v0.view(bits).numpy().copy()
        oracle_append(ko, vo, kn.view(bits).numpy(), vn.view(bits).numpy(), slots)
        oracle_copy_blocks(ko, vo, pairs)
        assert np.array_equal(cache.k_cache.cpu().view(bits).numpy(), ko)
        assert np.array_equal(cache.v_cache.cpu().view(bits).numpy(), vo)


def test_tiny_fp32_script(pa):
    """Tiny fp32 workload: lengths {1,16,17,45} in a 16-block seeded pool, one
    appended token per sequence, a fork of sequence 3 and one more token for the
    child (a copy-on-write of its shared partial block), then decode of all 5."""
    from paged_kv_cache_341_b200.cache import PagedKVCache
    w = workloads.get("tiny_fp32")
    lens0 = workloads.lengths(w)
    order = workloads.pool_order(w.num_blocks, w.seed)
    shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
    cache = PagedKVCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, torch.float32, 5,
                         w.max_blocks_per_seq, initial_free_order=order, fill=0.0)
    opool = OraclePool(w.num_blocks, w.block_size, order)
    otables, olens = [[] for _ in range(5)], [0] * 5
    ko = np.zeros(shape)
    vo = np.zeros(shape)

    def step(rows, seed):
        n = rows.stop - rows.start
        kn = workloads.randn((n, w.num_kv_heads, w.head_dim), "f32", seed)
        vn = workloads.randn((n, w.num_kv_heads, w.head_dim), "f32", seed + 1)
        slots, pairs = cache.reserve(rows)
        oslots, opairs = [], []
        for r in range(rows.start, rows.stop):
            slot, olens[r], src, dst = opool.reserve_slot(otables[r], olens[r])
            oslots.append(slot)
            if src >= 0:
                opairs.append((src, dst))
        assert list(slots) == oslots and [tuple(p) for p in pairs] == opairs
        cache.copy_blocks(torch.from_numpy(np.ascontiguousarray(pairs)).cuda())
        oracle_copy_blocks(ko, vo, opairs)
        cache.append(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda())
        oracle_append(ko, vo, kn.double().numpy(), vn.double().numpy(), oslots)
        return pairs

    # prefill token by token, one sequence after another
    seed = 500
    for r, n in enumerate(lens0):
        for _ in range(int(n)):
            step(slice(r, r + 1), seed)
            seed += 2
    step(slice(0, 4), 900)                          # one token each: lengths 2, 17, 18, 46
    cache.share(3, 4)                               # fork sequence 3 into row 4
    opool.fork(otables[3][: -(-olens[3] // w.block_size)])
    otables[4], olens[4] = list(otables[3]), olens[3]
    pairs = step(slice(4, 5), 950)                  # child writes at offset 14 of a shared block
    assert pairs.shape[0] == 1
    assert list(cache.lens) == [2, 17, 18, 46, 47] == olens
    refs, free = cache.pool.pa_pool_export()
    orefs, ofree = opool.export()
    assert list(refs) == orefs and list(free) == ofree and sum(r > 0 for r in refs) == 9
    cache.upload_tables()
    q_host = workloads.queries(w, 960, num_seqs=5)
    out = torch.empty((5, w.num_q_heads, w.head_dim), device="cuda")
    cache.attend(q_host.cuda(), out, w.scale)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    assert np.array_equal(cache.k_cache.cpu().numpy(), ko.astype(np.float32))
    assert np.array_equal(cache.v_cache.cpu().numpy(), vo.astype(np.float32))
    ref = oracle_decode(q_host.double().numpy(), ko, vo, otables, olens, w.scale)
    assert_close(out.cpu().numpy(), ref, "f32", "tiny script")


def test_device_checks_flag_bad_indices(pa):
    from paged_kv_cache_341_b200.cache import PagedKVCache
    cache = PagedKVCache(8, 16, 2, 64, torch.float32, 2, 4, fill=0.0)
    cache.allocate(0, 20)
    cache.allocate(1, 5)
    cache.tables[1, 0] = 8 + 5                     # outside the pool
    cache.upload_tables()
    q = torch.zeros(2, 2, 64, device="cuda")
    out = torch.empty_like(q)
    cache.attend(q, out, 0.125)
    assert pa.pa_device_error() == 1
    kn = torch.zeros(1, 2, 64, device="cuda")
    cache.append(kn, kn, torch.tensor([8 * 16 + 3], device="cuda"))
    assert pa.pa_device_error() == 3
    cache.copy_blocks(torch.tensor([[8, 1]], dtype=torch.int32, device="cuda"))
    assert pa.pa_device_error() == 4
    cache.d_lens.fill_(4 * 16 + 1)                 # beyond the table width
    cache.tables[1, 0] = 0
    cache.d_tables.copy_(torch.from_numpy(np.where(cache.tables < 0, 0, cache.tables)))
    cache.attend(q, out, 0.125)
    assert pa.pa_device_error() == 2
    # the context is still usable
    cache.upload_tables()
    cache.attend(q, out, 0.125)
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("partition", [0, 256])
def test_bounded_wait_runs_out_and_returns(pa, path, partition):
    """Every pipeline wait is bounded: with the test hook on, the producer of
    every decode CTA withholds its first stage, so the consumer's wait for it
    can only run out.  After 1 ms it does; every warp returns, the copies in
    flight land, the call completes and the device error word says 5
    (timeout).  The context stays usable: the next normal call is correct."""
    from paged_kv_cache_341_b200.cache import PagedKVCache
    lens = [1, 40, 700, 1500, 16, 0, 333]
    s, hq, hkv, d, bs = len(lens), 16, 4, 128, 16
    rng = np.random.default_rng(61)
    nb = sum(-(-n // bs) for n in lens) + 2
    mb = max(-(-n // bs) for n in lens) + 1
    cache = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, s, mb, initial_free_order=rng.permutation(nb))
    for row, n in enumerate(lens):
        cache.allocate(row, n)
    k_host, v_host = build_pool_contents((nb, bs, hkv, d), "bf16", cache.tables, lens, bs, 62)
    cache.k_cache.copy_(k_host)
    cache.v_cache.copy_(v_host)
    cache.upload_tables()
    q_host = workloads.randn((s, hq, d), "bf16", 63)
    q = q_host.cuda()
    scale = 1.0 / math.sqrt(d)
    ws = pa.decode_workspace(s, hq, d, mb, bs, partition)
    out = torch.zeros((s, hq, d), dtype=torch.bfloat16, device="cuda")
    assert pa.pa_device_error(reset=True) == 0
    pa.pa_debug_decode_stall(1_000_000)
    try:
        cache.attend(q, out, scale, partition, ws)
        code = pa.pa_device_error(reset=True)       # synchronises: the call has completed
    finally:
        pa.pa_debug_decode_stall(0)
    assert code == 5
    good = torch.full_like(out, float("nan"))
    cache.attend(q, good, scale, partition, ws)
    assert pa.pa_device_error() == 0
    ref = oracle_decode(q_host.double().numpy(), AsF64(k_host), AsF64(v_host), [list(r) for r in cache.tables],
                        lens, scale)
    assert_close(good.float().cpu().numpy(), ref, "bf16", "after a timed-out call")


def test_stall_hook_rejects_bad_bounds(pa):
    for bad in (-1, 10, 3_000_000_000):
        with pytest.raises(pa.PagedAttnError) as e:
            pa.pa_debug_decode_stall(bad)
        assert e.value.status == pa.PA_ERR_INVALID
    pa.pa_debug_decode_stall(0)
