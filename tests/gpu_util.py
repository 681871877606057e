"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads

TOL = 2e-3  # max-abs attention error against the binary64 oracle


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bfloat16 ulp at |x| (the rounding of a bf16 output)."""
    ax = np.maximum(np.abs(x), 1e-38)
    return 2.0 ** (np.floor(np.log2(ax)) - 8)


def gpu_cache_bytes(cache: kvq.KVCache):
    return [t.cpu().numpy() for t in (cache.k_codes, cache.v_codes, cache.k_params, cache.v_params)]


def oracle_cache_bytes(hc):
    return [hc.k_codes, hc.v_codes, hc.k_params.view(np.uint8), hc.v_params.view(np.uint8)]


def assert_same_cache(cache: kvq.KVCache, hc):
    names = ("k_codes", "v_codes", "k_params", "v_params")
    for name, g, o in zip(names, gpu_cache_bytes(cache), oracle_cache_bytes(hc)):
        if not np.array_equal(g, o):
            bad = np.flatnonzero(g != o)
            raise AssertionError(f"{name}: {bad.size} bytes differ, first at {bad[:8]}: "
                                 f"gpu {g[bad[:8]]} oracle {o[bad[:8]]}")


def both_quantize(ora, shape, k, v, pos, dtype_name=None):
    """Quantize the same inputs on the GPU and in the oracle."""
    B, Hkv, D, cap, bk, bv, G = shape
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, bk, bv, G)
    hc = ora.HostCache(B, Hkv, D, cap, bk, bv, G)
    append(ora, cache, hc, k, v, pos)
    return cache, hc


def append(ora, cache, hc, k, v, pos):
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    flags_o = hc.quantize_append(kb, vb, list(pos), dtype=dt)
    kvq.kvq_quantize_append(cache, k.cuda(), v.cuda(), torch.tensor(pos, dtype=torch.int32,
                                                                      device="cuda"))
    flags_g = kvq.kvq_device_error_flags()
    return flags_o, flags_g


def compare_attention(gpu_out: torch.Tensor, ref: np.ndarray, tol: float = TOL):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    if gpu_out.dtype == torch.bfloat16:
        bound = tol + bf16_half_ulp(ref)
    elif gpu_out.dtype == torch.float16:
        bound = tol + 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 11)
    else:
        bound = tol
    assert np.all(np.isfinite(g)), "non-finite output"
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (f"max err {err.max():.3e} at {worst}: gpu {g[worst]} "
                                  f"oracle {ref[worst]}")
    return float(err.max())
