"""The C-ABI library loads, exports every symbol include/pa.h declares, and
rejects bad arguments before touching the GPU (CPU only, no kernel launch)."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(built_library):
    names = declared_symbols()
    assert len(names) >= 16
    lib = ctypes.CDLL(built_library)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", built_library], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z_0-9]+)\b", out))
    assert set(names) <= exported
    # the binding declares a signature for each of them, no more, no less
    from paged_kv_cache_341_b200 import pa
    assert sorted(pa.SIGNATURES) == names


def test_library_is_built_for_sm100a(built_library):
    report = os.path.join(ROOT, "_build", "ptxas.txt")
    if not os.path.exists(report):
        pytest.skip("library shipped without its build report")
    text = open(report).read()
    assert "arch=compute_100a,code=sm_100a" in text
    assert "for 'sm_100a'" in text


def test_decode_rejects_bad_arguments_on_host(built_library):
    from paged_kv_cache_341_b200 import pa
    lib = pa._lib
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: validation fails first
    args = dict(q=fake, k=fake, v=fake, nb=16, tables=fake, mb=4, lens=fake, s=4, hq=2, hkv=2, d=64, bs=16,
                scale=0.125, p=0, ws=None, wsb=0, out=fake, dt=pa.PA_F32, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pa_decode_attention(a["q"], a["k"], a["v"], a["nb"], a["tables"], a["mb"], a["lens"], a["s"],
                                       a["hq"], a["hkv"], a["d"], a["bs"], a["scale"], a["p"], a["ws"], a["wsb"],
                                       a["out"], a["dt"], a["stream"])

    assert call(hq=3, hkv=2) == pa.PA_ERR_INVALID
    assert call(bs=24) == pa.PA_ERR_UNSUPPORTED
    assert call(p=24) == pa.PA_ERR_INVALID                  # not a multiple of block_size
    assert call(p=32) == pa.PA_ERR_INVALID                  # workspace missing
    assert call(dt=7) == pa.PA_ERR_INVALID
    assert call(q=ctypes.c_void_p((1 << 20) + 4)) == pa.PA_ERR_INVALID   # misaligned
    assert call(scale=float("nan")) == pa.PA_ERR_INVALID
    assert call(s=0) == pa.PA_OK                             # nothing to do, nothing launched
    assert "partition_size" in pa.pa_last_error() or call(p=24) == pa.PA_ERR_INVALID


def test_workspace_size_formula(built_library):
    from paged_kv_cache_341_b200 import pa
    def units(parts):
        return -(-8 * 64 * parts * 16 // 256) * 256
    assert pa.pa_decode_workspace_size(8, 64, 128, 1026, 32, 0) == 256 + units(1)
    np_ = -(-1026 * 32 // 512)
    assert pa.pa_decode_workspace_size(8, 64, 128, 1026, 32, 512) == 256 + units(np_) + 8 * 64 * np_ * (128 * 4 + 8)
    assert pa.pa_decode_workspace_size(0, 64, 128, 1026, 32, 512) == 0


def test_cache_ops_reject_bad_arguments_on_host(built_library):
    from paged_kv_cache_341_b200 import pa
    lib = pa._lib
    fake = ctypes.c_void_p(1 << 20)
    assert lib.pa_append_kv(fake, fake, fake, -1, fake, fake, 4, 16, 2, 64, pa.PA_F32, None) == pa.PA_ERR_INVALID
    assert lib.pa_append_kv(fake, fake, fake, 0, fake, fake, 4, 16, 2, 64, pa.PA_F32, None) == pa.PA_OK
    assert lib.pa_append_kv(fake, fake, fake, 3, fake, fake, 4, 16, 1, 3, pa.PA_F16, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_copy_blocks(fake, fake, fake, 0, 4, 16, 2, 64, pa.PA_BF16, None) == pa.PA_OK
    assert lib.pa_copy_blocks(None, fake, fake, 2, 4, 16, 2, 64, pa.PA_BF16, None) == pa.PA_ERR_INVALID


def test_binding_refuses_cpu_tensors(built_library):
    import torch
    from paged_kv_cache_341_b200 import pa
    x = torch.zeros(4, 2, 64)
    with pytest.raises(TypeError):
        pa.pa_decode_attention(x, torch.zeros(16, 16, 2, 64), torch.zeros(16, 16, 2, 64),
                               torch.zeros(4, 4, dtype=torch.int32), torch.zeros(4, dtype=torch.int32), 0.125,
                               torch.zeros(4, 2, 64))


def test_table_update_and_engine_reject_bad_arguments_on_host(built_library):
    import numpy as np
    from paged_kv_cache_341_b200 import pa
    lib = pa._lib
    fake = ctypes.c_void_p(1 << 20)
    # nothing to do -> OK without touching the device; bad sizes -> INVALID
    assert lib.pa_update_block_tables(fake, 4, 8, fake, 0, None, None, 0, None) == pa.PA_OK
    assert lib.pa_update_block_tables(fake, 4, 0, fake, 1, None, None, 0, None) == pa.PA_ERR_INVALID
    assert lib.pa_update_block_tables(fake, 4, 8, fake, 1, fake, fake, 5, None) == pa.PA_ERR_INVALID
    assert lib.pa_update_block_tables(None, 4, 8, None, 2, None, None, 0, None) == pa.PA_ERR_INVALID

    pool = pa.Pool(16, 16)
    tables = np.zeros((2, 4), np.int32)
    lens = np.zeros(2, np.int32)
    t32 = tables.ctypes.data_as(pa._p32)
    l32 = lens.ctypes.data_as(pa._p32)
    out = ctypes.c_void_p(123)

    def create(**kw):
        a = dict(pool=pool._h, tables=t32, lens=l32, s=2, mb=4, dt=fake, dl=fake, k=fake, v=fake, hq=4, hkv=2,
                 d=64, dtype=pa.PA_BF16, part=0)
        a.update(kw)
        return lib.pa_engine_create(a["pool"], a["tables"], a["lens"], a["s"], a["mb"], a["dt"], a["dl"], a["k"],
                                    a["v"], a["hq"], a["hkv"], a["d"], a["dtype"], a["part"], None,
                                    ctypes.byref(out))

    # every argument check runs before anything is allocated on the device
    assert create(pool=None) == pa.PA_ERR_INVALID and out.value is None
    assert create(s=0) == pa.PA_ERR_INVALID
    assert create(hq=3) == pa.PA_ERR_INVALID
    assert create(dtype=7) == pa.PA_ERR_INVALID
    assert create(k=ctypes.c_void_p((1 << 20) + 8)) == pa.PA_ERR_INVALID
    assert create(part=24) == pa.PA_ERR_INVALID
    assert create(part=-16) == pa.PA_ERR_INVALID
    assert lib.pa_engine_create(pool._h, t32, l32, 2, 4, fake, fake, fake, fake, 4, 2, 64, pa.PA_BF16, 0, None,
                                None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_step(None, 0, 1, fake, fake, fake, fake, 1.0, None, None, None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_join(None) == pa.PA_ERR_INVALID
    assert lib.pa_engine_synchronize(None) == pa.PA_ERR_INVALID
    lib.pa_engine_destroy(None)
    assert "pa_engine" in pa.pa_last_error()
