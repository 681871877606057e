"""Pins of the oracle's group quantizer.

The quantizer (group-wise asymmetric min-max, b-bit codes) is pinned against:
  * closed forms worked by hand (grids that quantize exactly, ties that round
    half to even, constant and -0 groups);
  * exact rational arithmetic: each code must be the nearest integer to the
    exact quotient (x - min) * (2^b - 1) / (max - min) unless that quotient is
    within binary32 rounding of a tie;
  * the per-element error bound |x - x^| <= scale/2 (plus the binary16
    rounding of the stored parameters), on every element of seeded inputs with
    the workloads' distributions;
  * code invariants: codes in [0, 2^b-1], the minimum maps to 0 and the
    maximum to 2^b-1 in every non-degenerate group; b=8 is near-identity.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from kv_cache_mixed_kvq_b200 import workloads


def f16(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_exact_grid(ora, bits):
    L = 2 ** bits - 1
    x = (np.arange(L + 1, dtype=np.float32) * 0.5 - 3.0)
    codes, s32, m32, s16, z16 = ora.quantize_group(x, bits)
    assert s32 == 0.5 and m32 == -3.0
    assert np.array_equal(codes, np.arange(L + 1))
    assert f16(s16) == 0.5 and f16(z16) == -3.0


def test_ties_round_half_even(ora):
    # range 3 at 2 bits -> scale 1, inv 1: quotients 0, .5, 1.5, 2.5, 3
    x = np.array([0.0, 0.5, 1.5, 2.5, 3.0], np.float32)
    codes, s32, m32, _, _ = ora.quantize_group(x, 2)
    assert (s32, m32) == (1.0, 0.0)
    assert codes.tolist() == [0, 0, 2, 2, 3]


def test_constant_group_is_degenerate_and_exact(ora):
    x = np.full(64, 1.25, np.float32)
    codes, s32, m32, s16, z16 = ora.quantize_group(x, 4)
    assert s32 == 0.0 and not codes.any()
    assert f16(s16) == 0.0 and f16(z16) == 1.25  # x^ = 0 * 0 + 1.25 exactly


def test_negative_zero_minimum_is_canonical(ora):
    x = np.array([-0.0, 1.0, 2.0, 3.0], np.float32)
    codes, s32, m32, s16, z16 = ora.quantize_group(x, 2)
    assert z16 == 0x0000  # +0, not the -0 pattern 0x8000
    assert codes.tolist() == [0, 1, 2, 3]


def test_signed_zero_extremes_give_positive_zero_params(ora):
    # all-zero group with mixed signs: range +0, scale +0, zero +0
    for x in ([-0.0, 0.0, -0.0], [0.0, -0.0], [-0.0, -0.0]):
        codes, s32, m32, s16, z16 = ora.quantize_group(np.array(x, np.float32), 4)
        assert (s16, z16) == (0x0000, 0x0000) and not codes.any()
    # negative group whose maximum is -0: range = 0 - mn
    codes, s32, m32, s16, z16 = ora.quantize_group(np.array([-3.0, -0.0], np.float32), 2)
    assert s32 == 1.0 and codes.tolist() == [0, 3]


def test_subnormal_range_degenerates(ora):
    # range 2^-140: scale is subnormal and 1/scale overflows -> all codes 0
    x = np.array([0.0, 2.0 ** -140], np.float32)
    codes, s32, _, _, _ = ora.quantize_group(x, 8)
    assert not codes.any()


def _exact_check(x, bits, codes):
    xs = [Fraction(float(v)) for v in x]
    mn, mx = min(xs), max(xs)
    L = 2 ** bits - 1
    if mx == mn:
        assert not codes.any()
        return
    for c, v in zip(codes.tolist(), xs):
        q = (v - mn) * L / (mx - mn)
        assert abs(c - q) <= Fraction(1, 2) + Fraction(2, 10 ** 4)
        frac = q - int(q)
        if abs(frac - Fraction(1, 2)) > Fraction(2, 10 ** 4):
            assert c == round(q)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_codes_are_nearest_levels_exact_rationals(ora, bits):
    rng = np.random.default_rng(bits)
    for trial in range(150):
        n = int(rng.choice([4, 7, 32, 64]))
        scale = 10.0 ** rng.uniform(-3, 3)
        x = (rng.standard_normal(n) * scale + rng.standard_normal() * scale).astype(np.float32)
        codes, *_ = ora.quantize_group(x, bits)
        _exact_check(x, bits, codes)


def _bound_check(x, bits, res):
    codes, s32, m32, s16, z16 = res
    L = 2 ** bits - 1
    assert codes.max() <= L
    if s32 == 0.0:
        return
    # min -> 0 and max -> L in every non-degenerate group
    assert codes[np.argmin(x)] == 0 and codes[np.argmax(x)] == L
    x64 = x.astype(np.float64)
    # fp32 parameters: half a step (plus a few binary32 roundings)
    e32 = np.abs(x64 - (codes * np.float64(s32) + np.float64(m32)))
    assert np.all(e32 <= s32 * (0.5 + 2e-4) + 1e-6 * np.abs(x64).max() * 2 ** -10)
    # stored binary16 parameters
    sc, z = f16(s16), f16(z16)
    deq = (codes.astype(np.float32) * np.float32(sc) + np.float32(z)).astype(np.float64)
    bound = s32 * (0.5 + 2e-4) + abs(m32 - z) + codes * abs(s32 - sc) + 2.0 ** -23 * np.abs(deq)
    assert np.all(np.abs(x64 - deq) <= bound + 1e-30)


@pytest.mark.parametrize("name", ["tiny", "llama3_8b", "qwen_mistral"])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_error_bound_on_workload_groups(ora, name, bits):
    w = workloads.WORKLOADS[name]
    k, v = workloads.make_kv(w, 64, seed=0, batch=1)
    for t in (k, v):
        arr = t.float().numpy().reshape(-1, w.group)
        for row in arr[:: max(1, arr.shape[0] // 128)]:
            _bound_check(row, bits, ora.quantize_group(row, bits))


def test_b8_near_identity(ora):
    w = workloads.WORKLOADS["llama3_8b"]
    _, v = workloads.make_kv(w, 32, seed=3, batch=1)
    for row in v.float().numpy().reshape(-1, 64):
        codes, s32, m32, s16, z16 = ora.quantize_group(row, 8)
        deq = codes * f16(s16) + f16(z16)
        rng_ = float(row.max() - row.min())
        assert np.abs(row - deq).max() <= rng_ / 510 * 1.001 + abs(m32 - f16(z16)) + \
            255 * abs(s32 - f16(s16)) + 1e-6


def test_bf16_input_matches_float_input(ora):
    # bfloat16 inputs are widened exactly; the append path must agree with
    # the group quantizer run on the widened values.
    w = workloads.WORKLOADS["llama3_8b"]
    k, v = workloads.make_kv(w, 16, seed=5, batch=1)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    cache = ora.HostCache(1, w.kv_heads, 128, 16, 4, 2, 64)
    assert cache.quantize_append(kb, vb, [0], dtype=dt) == 0
    kf = k.float().numpy()
    for h in range(w.kv_heads):
        for p in range(16):
            want = np.concatenate([ora.quantize_group(kf[0, h, p, g * 64:(g + 1) * 64], 4)[0]
                                   for g in range(2)])
            assert np.array_equal(cache.read_codes(0, 0, h, p), want)


@pytest.mark.parametrize("which,bits", [(0, 4), (1, 2), (1, 8)])
def test_cache_dequant_within_error_bound(ora, which, bits):
    # The dequantisation the attention oracle uses (codes read back from the
    # packed cache, times the stored binary16 scale, plus the stored zero)
    # must reconstruct the input to within half a quantization step.
    w = workloads.WORKLOADS["llama3_8b"]
    k, v = workloads.make_kv(w, 32, seed=9, batch=1)
    x = (k if which == 0 else v).float().numpy()
    cache = ora.HostCache(1, w.kv_heads, 128, 32, bits, bits, 64)
    cache.quantize_append(x if which == 0 else x * 0, x if which == 1 else x * 0, [0])
    params = (cache.k_params if which == 0 else cache.v_params).reshape(w.kv_heads, 32, 2, 2)
    for h in range(w.kv_heads):
        for p in range(32):
            deq = cache.dequant_row(which, 0, h, p).astype(np.float64)
            for g in range(2):
                s16 = f16(params[h, p, g, 0])
                xs = x[0, h, p, g * 64:(g + 1) * 64].astype(np.float64)
                err = np.abs(xs - deq[g * 64:(g + 1) * 64])
                L = 2 ** bits - 1
                assert err.max() <= s16 * (0.505 + L * 2.0 ** -11) + 2.0 ** -10 * np.abs(xs).max()
