"""GPU parity of the shared-prefix (cascade) decode against the oracle: the
result must equal plain attention over prefix ++ suffix for every sequence.
Tolerance as for every 16-bit cache: |gpu - ref| <= 2e-2 + 1e-2 |ref|."""

import math

import numpy as np
import pytest
import torch

from oracle import oracle_decode
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


@pytest.fixture(params=["umma", "pair", "mma"])
def prefix_path(request, monkeypatch):
    """Run a test on each prefix kernel: the SM-pair tcgen05 kernel (the default for head_dim 128; 64
    falls back to the one-SM kernel), the one-SM tcgen05 kernel and the mma.sync one."""
    monkeypatch.setenv("PA_PREFIX_PATH", request.param)
    return request.param


def cascade_case(dtype, hkv, d, bs, prefix_len, suffixes, seed):
    """A pool whose sequences share prefix_len tokens copy-on-write, then hold
    their own suffixes; returns the cache and its host K/V contents."""
    from paged_kv_cache_341_b200.cache import PagedKVCache
    rng = np.random.default_rng(seed)
    s = len(suffixes)
    pblocks = prefix_len // bs
    sblocks = [-(-n // bs) for n in suffixes]
    nb = pblocks + sum(sblocks) + 4
    mb = pblocks + max(sblocks + [1]) + 1
    cache = PagedKVCache(nb, bs, hkv, d, TORCH[dtype], s, mb, initial_free_order=rng.permutation(nb))
    if prefix_len:
        cache.allocate(0, prefix_len)
        for r in range(1, s):
            cache.share(0, r)
    for r, n in enumerate(suffixes):
        if n:
            cache.tables[r, pblocks:pblocks + sblocks[r]] = cache.pool.pa_pool_alloc(sblocks[r])
        cache.lens[r] = prefix_len + n
    k_host, v_host = build_pool_contents((nb, bs, hkv, d), dtype, cache.tables, cache.lens, bs, seed)
    cache.k_cache.copy_(k_host)
    cache.v_cache.copy_(v_host)
    cache.upload_tables()
    return cache, k_host, v_host, mb


def run_cascade(pa, dtype, hq, hkv, d, bs, prefix_len, suffixes, partition, seed, q_scale=1.0):
    s = len(suffixes)
    pblocks = prefix_len // bs
    cache, k_host, v_host, mb = cascade_case(dtype, hkv, d, bs, prefix_len, suffixes, seed)
    q_host = workloads.randn((s, hq, d), dtype, seed + 2)
    if q_scale != 1.0:
        q_host = (q_host.float() * q_scale).to(TORCH[dtype])
    q = q_host.cuda()
    scale = 1.0 / math.sqrt(d)
    out = torch.full((s, hq, d), float("nan"), dtype=TORCH[dtype], device="cuda")
    prefix_ids = cache.d_tables[0, :pblocks].contiguous()
    suffix_tables = cache.d_tables[:, pblocks:]
    suffix_lens = cache.d_lens - prefix_len
    pa.pa_decode_attention_shared_prefix(q, cache.k_cache, cache.v_cache, prefix_ids, prefix_len, suffix_tables,
                                         suffix_lens, scale, out, partition_size=partition)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    ref = oracle_decode(q_host.double().numpy(), AsF64(k_host), AsF64(v_host),
                        [list(r) for r in cache.tables], [int(x) for x in cache.lens], scale)
    plain = torch.empty_like(out)
    ws = pa.decode_workspace(s, hq, d, mb, bs, partition)
    cache.attend(q, plain, scale, partition, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), ref, plain.float().cpu().numpy()


SUFFIXES = [0, 1, 15, 16, 17, 100, 33]

# pa_debug_last_prefix_kernel per path; the SM-pair kernel takes head_dim 128
# only (64 falls back to the one-SM kernel), and on a B200 it always launches
LAUNCHED = {"pair": 1, "umma": 2, "mma": 3}


def check_launched(pa, prefix_path, d):
    want = LAUNCHED[prefix_path] if not (prefix_path == "pair" and d != 128) else LAUNCHED["umma"]
    assert pa.pa_debug_last_prefix_kernel() == want, (prefix_path, d, pa.pa_debug_last_prefix_kernel())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (16, 4), (16, 2)])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("prefix_len", [32, 1056, 1088])
@pytest.mark.parametrize("partition", [0, 64])
def test_shared_prefix_matches_oracle(pa, prefix_path, dtype, d, hq, hkv, bs, prefix_len, partition):
    # 1056 = 1024 + 32: the second slice ends in a 32-token tile; 1088 ends on a full one
    gpu, ref, plain = run_cascade(pa, dtype, hq, hkv, d, bs, prefix_len, SUFFIXES, partition,
                                  seed=prefix_len + bs + hq + d + partition)
    check_launched(pa, prefix_path, d)
    tag = "%s dtype=%s d=%d hq=%d hkv=%d bs=%d prefix=%d p=%d" % (prefix_path, dtype, d, hq, hkv, bs, prefix_len,
                                                                  partition)
    assert_close(gpu, ref, dtype, tag)
    assert_close(gpu, plain.astype(np.float64), dtype, tag + " vs plain call")


@pytest.mark.parametrize("nseq", [70, 50, 64])
def test_many_sequences_and_row_tiles(pa, prefix_path, nseq):
    # x 4 query rows per KV head: 280 = tiles of 128, 128 and 24; 200 = 128 and
    # 72 (a partly filled second tile of a CTA); 256 = exactly two full tiles
    rng = np.random.default_rng(5)
    suffixes = [int(x) for x in rng.integers(0, 600, size=nseq)]
    gpu, ref, _ = run_cascade(pa, "bf16", 32, 8, 128, 16, 2048 + 64, suffixes, 512, seed=6 + nseq)
    check_launched(pa, prefix_path, 128)
    assert_close(gpu, ref, "bf16", "%d sequences" % nseq)


def test_prefix_of_more_than_64_slices(pa, prefix_path):
    # 33,280 prefix tokens = 65 slices of 512 plus the suffix partitions: the
    # merge reads the (m, l) pairs of slots 64 and up in a second sweep
    gpu, ref, plain = run_cascade(pa, "bf16", 8, 2, 128, 16, 33280, [0, 5, 300, 77], 256, seed=9)
    check_launched(pa, prefix_path, 128)
    assert_close(gpu, ref, "bf16", "%s, 65 prefix slices" % prefix_path)
    assert_close(gpu, plain.astype(np.float64), "bf16", "%s, 65 prefix slices vs plain call" % prefix_path)


def test_large_scores_rescale_in_tensor_memory(pa, prefix_path):
    # queries scaled up so the running maximum moves by more than 2^8 between
    # tiles: the tcgen05 kernel rescales O inside tensor memory
    gpu, ref, _ = run_cascade(pa, "bf16", 16, 4, 128, 16, 1024 + 512, [3, 0, 40], 0, seed=8, q_scale=12.0)
    check_launched(pa, prefix_path, 128)
    assert_close(gpu, ref, "bf16", "large scores")


def test_back_to_back_calls_on_a_stream(pa, prefix_path):
    # The prefix kernel runs on the library's side stream, forked from the
    # caller's stream and joined back before the merge.  Three calls queued on
    # a non-default stream without a sync, sharing one workspace, each with
    # queries written on that stream just before it: every output must be its
    # own call's.
    dtype, hq, hkv, d, bs, prefix_len = "bf16", 32, 8, 128, 16, 2048 + 64
    rng = np.random.default_rng(11)
    suffixes = [int(x) for x in rng.integers(0, 300, size=40)]
    s, pblocks = len(suffixes), prefix_len // bs
    cache, k_host, v_host, _ = cascade_case(dtype, hkv, d, bs, prefix_len, suffixes, 12)
    scale = 1.0 / math.sqrt(d)
    prefix_ids = cache.d_tables[0, :pblocks].contiguous()
    suffix_tables = cache.d_tables[:, pblocks:]
    suffix_lens = (cache.d_lens - prefix_len).contiguous()
    q_hosts = [workloads.randn((s, hq, d), dtype, 20 + i) for i in range(3)]
    q_srcs = [q.cuda() for q in q_hosts]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    ws = None
    outs = []
    with torch.cuda.stream(stream):
        for i in range(3):
            q_i = torch.empty_like(q_srcs[i])
            q_i.copy_(q_srcs[i])          # written on the stream right before the call
            out = torch.full((s, hq, d), float("nan"), dtype=TORCH[dtype], device="cuda")
            ws = pa.pa_decode_attention_shared_prefix(q_i, cache.k_cache, cache.v_cache, prefix_ids, prefix_len,
                                                      suffix_tables, suffix_lens, scale, out, partition_size=512,
                                                      workspace=ws, stream=stream)
            outs.append(out)
    stream.synchronize()
    assert pa.pa_device_error() == 0
    check_launched(pa, prefix_path, d)
    for i in range(3):
        ref = oracle_decode(q_hosts[i].double().numpy(), AsF64(k_host), AsF64(v_host),
                            [list(r) for r in cache.tables], [int(x) for x in cache.lens], scale)
        assert_close(outs[i].float().cpu().numpy(), ref, dtype, "%s call %d" % (prefix_path, i))


def test_calls_from_two_host_threads(pa):
    # Two host threads, each with its own stream, workspace and queries, call
    # the cascade at the same time; the library's side stream (and its fork and
    # join events) is shared, so each call's fork, prefix launch and join must
    # stay together.  Every output must be its own call's.
    import threading
    dtype, hq, hkv, d, bs, prefix_len = "bf16", 16, 4, 128, 16, 1024 + 64
    rng = np.random.default_rng(13)
    suffixes = [int(x) for x in rng.integers(0, 200, size=24)]
    s, pblocks = len(suffixes), prefix_len // bs
    cache, k_host, v_host, _ = cascade_case(dtype, hkv, d, bs, prefix_len, suffixes, 14)
    scale = 1.0 / math.sqrt(d)
    prefix_ids = cache.d_tables[0, :pblocks].contiguous()
    suffix_tables = cache.d_tables[:, pblocks:]
    suffix_lens = (cache.d_lens - prefix_len).contiguous()
    q_hosts = [workloads.randn((s, hq, d), dtype, 30 + i) for i in range(2)]
    qs = [q.cuda() for q in q_hosts]
    torch.cuda.synchronize()
    outs = [[], []]
    errors = []

    def worker(i):
        try:
            stream = torch.cuda.Stream()
            ws = None
            with torch.cuda.stream(stream):
                for _ in range(20):
                    out = torch.full((s, hq, d), float("nan"), dtype=TORCH[dtype], device="cuda")
                    ws = pa.pa_decode_attention_shared_prefix(qs[i], cache.k_cache, cache.v_cache, prefix_ids,
                                                              prefix_len, suffix_tables, suffix_lens, scale, out,
                                                              partition_size=256, workspace=ws, stream=stream)
                    outs[i].append(out)
            stream.synchronize()
        except Exception as e:      # reported on the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert pa.pa_device_error() == 0
    for i in range(2):
        ref = oracle_decode(q_hosts[i].double().numpy(), AsF64(k_host), AsF64(v_host),
                            [list(r) for r in cache.tables], [int(x) for x in cache.lens], scale)
        first = outs[i][0].float().cpu().numpy()
        assert_close(first, ref, dtype, "thread %d" % i)
        for j, o in enumerate(outs[i][1:]):
            assert np.array_equal(o.float().cpu().numpy(), first), (i, j)


def test_zero_prefix_is_the_plain_call(pa):
    gpu, ref, plain = run_cascade(pa, "bf16", 8, 2, 128, 16, 0, [5, 40], 0, seed=7)
    assert_close(gpu, ref, "bf16", "no prefix")
    assert np.array_equal(gpu, plain)


def test_rejects_bad_arguments(pa):
    q = torch.zeros(2, 8, 128, dtype=torch.float32, device="cuda")
    kc = torch.zeros(4, 16, 2, 128, dtype=torch.float32, device="cuda")
    tables = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    lens = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_decode_attention_shared_prefix(q, kc, kc, tables[0], 16, tables, lens, 0.1, q)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    qb, kb = q.bfloat16(), kc.bfloat16()
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_decode_attention_shared_prefix(qb, kb, kb, tables[0], 24, tables, lens, 0.1, qb)
    assert e.value.status == pa.PA_ERR_INVALID
