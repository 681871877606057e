"""The C-ABI library on a machine without a GPU: it loads, exports every
entry point its header declares, sizes caches, and rejects invalid arguments
on the host before any CUDA call (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import kv_cache_mixed_kvq_b200 as kvq

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "kvq.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("kvq_quantize_append", "kvq_decode_attention", "kvq_cache_bytes",
              "kvq_decode_workspace_bytes", "kvq_device_error_flags", "kvq_last_device_error",
              "kvq_decode_attention_static", "kvq_append_decode_attention", "kvq_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = kvq.library()
    for name in _declared():
        assert hasattr(lib, name), name


def test_cache_bytes_and_memory_claim():
    # "Key contributions": K4V2 takes 25% less KV-cache memory than K4V4
    cb = kvq.kvq_cache_bytes
    k4v2 = cb(1, 8, 128, 4096, 4, 2, 64, kvq.KVQ_K_CODES) + cb(1, 8, 128, 4096, 4, 2, 64, kvq.KVQ_V_CODES)
    k4v4 = cb(1, 8, 128, 4096, 4, 4, 64, kvq.KVQ_K_CODES) + cb(1, 8, 128, 4096, 4, 4, 64, kvq.KVQ_V_CODES)
    assert k4v2 / k4v4 == 0.75
    params = cb(1, 8, 128, 4096, 4, 2, 64, kvq.KVQ_K_PARAMS) * 2
    assert (k4v2 + params) / (k4v4 + params) == pytest.approx(7 / 9)
    # bytes per token-head at D=128, G=64: K4 64 + V2 32 + 2 * 8 params = 112
    assert (k4v2 + params) / (8 * 4096) == 112


@pytest.mark.parametrize("args", [
    (0, 8, 128, 64, 4, 2, 64), (1, 8, 96, 64, 4, 2, 64), (1, 8, 128, 40, 4, 2, 64),
    (1, 8, 128, 64, 3, 2, 64), (1, 8, 128, 64, 4, 1, 64), (1, 8, 64, 64, 4, 2, 128),
    (1, 8, 128, 64, 4, 2, 48),
])
def test_cache_bytes_rejects_bad_shapes(args):
    assert kvq.kvq_cache_bytes(*args, kvq.KVQ_K_CODES) == 0


def _desc(**kw):
    d = dict(batch=1, kv_heads=2, head_dim=128, capacity=64, bits_k=4, bits_v=2, group=64,
             flags=0, group_v=0, reserved=0, k_codes=0x1000, v_codes=0x2000, k_params=0x3000, v_params=0x4000,
             page_size=0, num_pages=0, block_table=None)
    d.update(kw)
    return kvq.KvqCacheDesc(*d.values())


def test_validate_cache_host_only():
    lib = kvq.library()
    assert lib.kvq_validate_cache(ctypes.byref(_desc())) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(_desc(k_codes=0x1008))) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_validate_cache(ctypes.byref(_desc(v_params=0))) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_validate_cache(ctypes.byref(_desc(flags=kvq.KVQ_FLAG_ROTATE_KEYS))) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(_desc(flags=4))) == kvq.KVQ_ERR_INVALID_ARG
    # paged layout: power-of-two pages of >= 32 positions dividing capacity,
    # a pool of >= 1 page and an aligned block table; none of it without the flag
    paged = dict(flags=kvq.KVQ_FLAG_PAGED, page_size=32, num_pages=5, block_table=0x5000)
    assert lib.kvq_validate_cache(ctypes.byref(_desc(**paged))) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(_desc(**dict(paged, page_size=64)))) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(
        _desc(**dict(paged, flags=3)))) == kvq.KVQ_OK  # with key rotation
    for bad in (dict(page_size=16), dict(page_size=48), dict(page_size=128), dict(page_size=0),
                dict(num_pages=0), dict(block_table=None), dict(block_table=0x5002)):
        assert lib.kvq_validate_cache(ctypes.byref(_desc(**dict(paged, **bad)))) == \
            kvq.KVQ_ERR_INVALID_ARG, bad
    for stray in (dict(page_size=32), dict(num_pages=1), dict(block_table=0x5000)):
        assert lib.kvq_validate_cache(ctypes.byref(_desc(**stray))) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_validate_cache(ctypes.byref(_desc(reserved=1))) == kvq.KVQ_ERR_INVALID_ARG
    # value groups: equal or coarser than the keys' (group 64 here)
    assert lib.kvq_validate_cache(ctypes.byref(_desc(group_v=128))) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(_desc(group_v=64))) == kvq.KVQ_OK
    assert lib.kvq_validate_cache(ctypes.byref(_desc(group_v=32))) == kvq.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_validate_cache(ctypes.byref(_desc(group_v=48))) == kvq.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_validate_cache(ctypes.byref(_desc(bits_v=3))) == kvq.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_validate_cache(ctypes.byref(_desc(capacity=24))) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_validate_cache(None) == kvq.KVQ_ERR_INVALID_ARG


def test_quantize_append_rejects_before_launch():
    lib = kvq.library()
    d = _desc()
    q = lib.kvq_quantize_append
    assert q(ctypes.byref(_desc(group=48)), 0x10, 0x20, 1, 0x30, 1, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert q(ctypes.byref(d), None, 0x20, 1, 0x30, 1, None) == kvq.KVQ_ERR_INVALID_ARG
    assert q(ctypes.byref(d), 0x18, 0x20, 1, 0x30, 1, None) == kvq.KVQ_ERR_INVALID_ARG
    assert q(ctypes.byref(d), 0x10, 0x20, 7, 0x30, 1, None) == kvq.KVQ_ERR_INVALID_ARG
    assert q(ctypes.byref(d), 0x10, 0x20, 1, 0x30, 65, None) == kvq.KVQ_ERR_INVALID_ARG
    assert q(ctypes.byref(d), 0x10, 0x20, 1, 0x31, 1, None) == kvq.KVQ_ERR_INVALID_ARG
    # n_new == 0 is a no-op that touches nothing
    assert q(ctypes.byref(d), 0x10, 0x20, 1, 0x30, 0, None) == kvq.KVQ_OK


def test_decode_rejects_before_launch():
    lib = kvq.library()
    d = _desc()
    f = lib.kvq_decode_attention
    ok = dict(q=0x100, qt=1, hq=8, lens=0x200, maxlen=64, scale=0.0, out=0x300, ot=1, ws=0x400,
              wsb=1 << 20)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(ctypes.byref(a.pop("desc", d)), a["q"], a["qt"], a["hq"], a["lens"], a["maxlen"],
                 a["scale"], a["out"], a["ot"], a["ws"], a["wsb"], None)

    assert call(hq=7) == kvq.KVQ_ERR_INVALID_ARG          # not a multiple of Hkv
    assert call(hq=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(q=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(q=0x104) == kvq.KVQ_ERR_INVALID_ARG       # misaligned
    assert call(qt=9) == kvq.KVQ_ERR_INVALID_ARG
    assert call(ot=-1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(lens=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(maxlen=-1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(scale=float("nan")) == kvq.KVQ_ERR_INVALID_ARG
    assert call(desc=_desc(head_dim=80)) == kvq.KVQ_ERR_UNSUPPORTED


def test_strerror():
    assert kvq.kvq_strerror(kvq.KVQ_OK) == "ok"
    assert "workspace" in kvq.kvq_strerror(kvq.KVQ_ERR_WORKSPACE)
    assert kvq.kvq_strerror(99) == "unknown status"


def test_fused_append_rejects_before_launch():
    lib = kvq.library()
    d = _desc()
    f = lib.kvq_append_decode_attention

    def call(k=0x500, v=0x600, dt=1, n=1, hq=8, q=0x100):
        return f(ctypes.byref(d), k, v, dt, n, q, 1, hq, 0x200, 64, 0.0, 0x300, 1, 0x400,
                 1 << 20, None)

    assert call(n=-1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(k=None) == kvq.KVQ_ERR_INVALID_ARG
    assert call(v=0x608) == kvq.KVQ_ERR_INVALID_ARG      # misaligned
    assert call(dt=5) == kvq.KVQ_ERR_INVALID_ARG
    assert call(hq=7) == kvq.KVQ_ERR_INVALID_ARG         # decode checks still apply
    assert call(q=0) == kvq.KVQ_ERR_INVALID_ARG


def test_wait_timeout_knob_is_validated_on_the_host():
    lib = kvq.library()
    assert lib.kvq_debug_inject_wait_timeout(0, 10) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_debug_inject_wait_timeout(2, 1_000_000) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_debug_inject_wait_timeout(0, 2_000_000_000) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_debug_inject_wait_timeout(-1, 0) == kvq.KVQ_OK
