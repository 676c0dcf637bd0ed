"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, sizes buffers, and rejects bad arguments on
the host before touching the device."""

import ctypes
import os
import re

import pytest

from h2o_kv_cache_attn_b200 import binding as hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"H2OKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_loads_and_exports_every_declared_symbol():
    lib = hb.load()
    declared = header_symbols()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(lib, name), name
    assert set(hb.EXPORTED) <= set(declared)
    assert hb.h2okv_abi_version() == 1


def desc(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, capacity=32768, max_chunk=1024,
                q_dtype=hb.BF16, kv_dtype=hb.BF16)
    base.update(kw)
    return hb.CacheDesc(**base)


def test_query_sizes_by_dtype():
    slots = 8 * 32768
    for kv, row in ((hb.BF16, 256), (hb.I8, 128), (hb.I4, 64)):
        s = hb.kv_cache_query_sizes(desc(kv_dtype=kv))
        assert s["keys"] == s["values"] == slots * row
        assert s["token_pos"] == s["scores"] == slots * 4
        assert s["k_scales"] == s["v_scales"] == (slots * 2 if kv != hb.BF16 else 0)
        assert s["workspace"] >= 32 * 1024 * 4  # one log-sum-exp per query row
        if kv == hb.BF16:  # tensor-core path: per-row-tile summed weights
            assert s["workspace"] >= 32 * 8 * 32768 * 4
        assert s["workspace"] % 256 == 0
    s = hb.kv_cache_query_sizes(desc(q_dtype=hb.F32, kv_dtype=hb.F32, head_dim=64))
    assert s["keys"] == slots * 64 * 4


@pytest.mark.parametrize("bad", [
    dict(n_q_heads=30), dict(head_dim=100), dict(head_dim=264), dict(capacity=0),
    dict(capacity=70000), dict(max_chunk=0), dict(q_dtype=7), dict(kv_dtype=9),
    dict(q_dtype=hb.BF16, kv_dtype=hb.F32), dict(q_dtype=hb.F32, kv_dtype=hb.I8),
    dict(batch=0)])
def test_bad_descriptions_rejected(bad):
    with pytest.raises(hb.H2OKVError) as e:
        hb.kv_cache_query_sizes(desc(**bad))
    assert e.value.code == hb.ERR_INVALID_ARG
    assert hb.h2okv_last_error() != ""


def test_create_rejects_missing_or_misaligned_buffers():
    lib = hb.load()
    d = desc(capacity=256, max_chunk=64)
    h = ctypes.c_void_p()
    bufs = hb.CacheBuffers(None, None, None, None, None, None, None)
    assert lib.kv_cache_create(ctypes.byref(d), ctypes.byref(bufs), None, ctypes.byref(h)) == hb.ERR_INVALID_ARG
    fake = 0x10000000
    bufs = hb.CacheBuffers(fake + 4, fake, None, None, fake, fake, fake)
    assert lib.kv_cache_create(ctypes.byref(d), ctypes.byref(bufs), None, ctypes.byref(h)) == hb.ERR_INVALID_ARG
    assert "aligned" in hb.h2okv_last_error()
    dq = desc(capacity=256, max_chunk=64, kv_dtype=hb.I8)
    bufs = hb.CacheBuffers(fake, fake, None, None, fake, fake, fake)
    assert lib.kv_cache_create(ctypes.byref(dq), ctypes.byref(bufs), None, ctypes.byref(h)) == hb.ERR_INVALID_ARG


def test_calls_on_null_handle_and_bad_sizes():
    lib = hb.load()
    assert lib.h2o_evict_insert(None, None, None, None, 1, 0, None, None) == hb.ERR_INVALID_ARG
    assert lib.attn_chunk_with_scoresum(None, None, 1, 0, None, None, None, None, None) == hb.ERR_INVALID_ARG
    assert lib.kv_cache_quantize(hb.BF16, None, 4, 128, None, None, None) == hb.ERR_INVALID_ARG
    assert lib.kv_cache_quantize(hb.I8, None, 4, 100, None, None, None) == hb.ERR_INVALID_ARG
    assert lib.kv_cache_quantize(hb.I8, None, 0, 128, None, None, None) == hb.OK
    assert lib.kv_cache_destroy(None) == hb.OK


def test_package_has_no_oracle_dependency():
    # the product package must not reach into the test oracle
    pkg = os.path.join(ROOT, "h2o_kv_cache_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), f
                assert "oracle/" not in src, f
