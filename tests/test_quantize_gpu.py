"""GPU quantize-append vs the oracle: all four cache arrays bit-exact."""
import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import append, assert_same_cache, both_quantize

pytestmark = pytest.mark.gpu

SHAPES = [(D, bk, bv, G) for D in (64, 128) for bk in (2, 4, 8) for bv in (2, 4, 8)
          for G in (32, 64, 128) if G <= D]


def _inputs(B, Hkv, n, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    centre = torch.randn(Hkv, 1, D, generator=g) * 2
    k = (centre + torch.randn(B, Hkv, n, D, generator=g)) * (1 + 9 * (torch.rand(D, generator=g) < 0.03))
    v = torch.randn(B, Hkv, n, D, generator=g)
    return k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("D,bk,bv,G", SHAPES)
def test_full_tiles_all_shapes(ora, D, bk, bv, G):
    B, Hkv, n = 2, 3, 48
    k, v = _inputs(B, Hkv, n, D, torch.bfloat16, seed=D + 10 * bk + 100 * bv + G)
    cache, hc = both_quantize(ora, (B, Hkv, D, 64, bk, bv, G), k, v, [0, 16])
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_input_dtypes(ora, dtype):
    k, v = _inputs(2, 2, 33, 128, dtype, seed=7)
    cache, hc = both_quantize(ora, (2, 2, 128, 64, 4, 2, 64), k, v, [0, 5])
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("steps", [[(0, 1)], [(5, 1), (6, 3)], [(15, 2)], [(3, 29), (32, 16)],
                                   [(0, 16), (16, 1), (17, 15), (32, 31)]])
def test_appends_at_any_alignment(ora, steps):
    B, Hkv, D, cap = 2, 2, 128, 96
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    hc = ora.HostCache(B, Hkv, D, cap, 4, 2, 64)
    for i, (pos, n) in enumerate(steps):
        k, v = _inputs(B, Hkv, n, D, torch.bfloat16, seed=100 + i)
        fo, fg = append(ora, cache, hc, k, v, [pos, pos + 1])
        assert fo == 0 and fg == 0
        assert_same_cache(cache, hc)


def test_degenerate_and_signed_zero_groups(ora):
    B, Hkv, D, n = 1, 1, 64, 16
    k = torch.zeros(B, Hkv, n, D)
    k[0, 0, 0, :32] = 3.25              # constant group
    k[0, 0, 1, :] = -0.0                # all -0
    k[0, 0, 2, ::2] = -0.0              # mixed zeros
    k[0, 0, 3, :32] = torch.linspace(-4, 0, 32)
    k[0, 0, 3, 31] = -0.0               # maximum is -0
    k[0, 0, 4, ::2] = 2.0 ** -140           # subnormal range: 1/scale overflows
    k[0, 0, 5, :32] = 65504.0
    k[0, 0, 5, 0] = -65504.0            # full binary16 range
    k[0, 0, 6] = torch.arange(64) * 0.5 - 3  # exact grid
    v = -k
    for dtype in (torch.float32, torch.bfloat16):
        cache, hc = both_quantize(ora, (B, Hkv, D, 16, 4, 2, 32), k.to(dtype), v.to(dtype), [0])
        assert_same_cache(cache, hc)
        cache, hc = both_quantize(ora, (B, Hkv, D, 16, 8, 8, 32), k.to(dtype), v.to(dtype), [0])
        assert_same_cache(cache, hc)


def test_ties_and_random_magnitudes(ora):
    g = torch.Generator().manual_seed(3)
    B, Hkv, D, n = 2, 2, 128, 32
    # values on a half-step grid produce many exact .5 ties
    k = torch.randint(-20, 20, (B, Hkv, n, D), generator=g).float() * 0.25
    v = torch.randn(B, Hkv, n, D, generator=g) * torch.logspace(-4, 4, n)[None, None, :, None]
    for bits in ((2, 2), (4, 4), (8, 8)):
        cache, hc = both_quantize(ora, (B, Hkv, D, 32, *bits, 32), k, v.float(), [0, 0])
        assert_same_cache(cache, hc)


def test_capacity_and_bad_pos_are_flagged_and_skipped(ora):
    B, Hkv, D, cap = 3, 1, 64, 32
    k, v = _inputs(B, Hkv, 4, D, torch.bfloat16, seed=9)
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 32)
    hc = ora.HostCache(B, Hkv, D, cap, 4, 2, 32)
    fo, fg = append(ora, cache, hc, k, v, [30, 0, -2])
    assert fo == (kvq.KVQ_DEVERR_CAPACITY | kvq.KVQ_DEVERR_BAD_POS)
    assert fg == fo
    assert_same_cache(cache, hc)
    assert kvq.kvq_device_error_flags() == 0  # reading clears


def test_workload_slices_bit_exact(ora):
    # the workloads' own distributions (outlier channels, bf16/fp32)
    for name in ("tiny", "llama3_8b", "qwen_mistral"):
        w = workloads.WORKLOADS[name]
        k, v = workloads.make_kv(w, 80, seed=1, batch=2)
        for bk, bv in w.bits:
            cache, hc = both_quantize(ora, (2, w.kv_heads, w.head_dim, 96, bk, bv, w.group),
                                      k, v, [0, 7])
            assert_same_cache(cache, hc)
