"""Pins of the oracle's number conversions against library routines.

binary32 -> binary16 (round to nearest even) is pinned against numpy's
float16 cast; binary16 -> binary32 on all 65536 bit patterns; bfloat16 ->
binary32 against torch's bfloat16.
"""
import numpy as np
import pytest
import torch


def _np_f16_bits(x: float) -> int:
    with np.errstate(over="ignore"):
        return int(np.array([x], np.float32).astype(np.float16).view(np.uint16)[0])


EDGE = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e9, -1e9,
        2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -26, 1.5 * 2.0 ** -24,
        2.5 * 2.0 ** -24, 6.1e-5, 6.0e-8, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
        2048.0 + 1.0, 2048.0 + 3.0, 0.1, 1.0 / 3.0, float("inf"), -float("inf")]


@pytest.mark.parametrize("x", EDGE)
def test_f32_to_f16_edges(ora, x):
    assert ora.f32_to_f16_bits(x) == _np_f16_bits(x)


def test_f32_to_f16_random_patterns(ora):
    rng = np.random.default_rng(1)
    # random finite binary32 bit patterns concentrated around binary16's range
    mags = rng.uniform(-30, 17, 20000)
    vals = (np.sign(rng.standard_normal(20000)) * 2.0 ** mags).astype(np.float32)
    pats = rng.integers(0, 2 ** 32, 5000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    vals = np.concatenate([vals, pats[np.isfinite(pats)]])
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([ora.f32_to_f16_bits(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)


def test_f32_to_f16_nan(ora):
    h = ora.f32_to_f16_bits(float("nan"))
    assert (h & 0x7C00) == 0x7C00 and (h & 0x3FF) != 0


def test_f16_to_f32_all_patterns(ora):
    pats = np.arange(65536, dtype=np.uint16)
    want = pats.view(np.float16).astype(np.float32)
    got = np.array([ora.f16_bits_to_f32(int(p)) for p in pats], np.float32)
    finite = np.isfinite(want) | np.isinf(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.all(np.isnan(got[~finite]))


def test_bf16_to_f32(ora):
    rng = np.random.default_rng(2)
    pats = rng.integers(0, 65536, 20000).astype(np.uint16)
    want = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([ora.bf16_bits_to_f32(int(p)) for p in pats], np.float32)
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
