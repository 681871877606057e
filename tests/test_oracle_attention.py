"""Pins of the oracle's decode attention (binary64 on the dequantised cache).

  * closed forms: one token -> its value row; equal keys -> mean of values;
    one dominant score -> that token's value row;
  * brute force with pure-Python loops (math.exp) on tiny inputs;
  * a library routine (numpy matmul + scipy softmax) on larger inputs;
  * grouped-query mapping (query head hq reads kv head hq // (Hq/Hkv)),
    default scale 1/sqrt(D), empty sequences and length clamping;
  * the unquantised attention oracle against the same library routine.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax

from kv_cache_mixed_kvq_b200 import workloads


def _filled_cache(ora, B, Hkv, D, T, bk=4, bv=2, G=64, seed=0, cap=None):
    rng = np.random.default_rng(seed)
    cap = cap or (T + 15) // 16 * 16
    cache = ora.HostCache(B, Hkv, D, cap, bk, bv, G)
    k = (rng.standard_normal((B, Hkv, T, D)) * 2).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    assert cache.quantize_append(k, v, [0] * B) == 0
    return cache, k, v


def _deq(cache, b, h, n):
    return (cache.dequant_slot(0, b, h, n).astype(np.float64),
            cache.dequant_slot(1, b, h, n).astype(np.float64))


def test_single_token_returns_its_value(ora):
    cache, _, _ = _filled_cache(ora, 1, 1, 64, 1, G=32)
    q = np.random.default_rng(1).standard_normal((1, 1, 64)).astype(np.float32)
    out, flags = cache.decode_attention(q, 1, [1])
    assert flags == 0
    _, vh = _deq(cache, 0, 0, 1)
    assert np.array_equal(out[0, 0], vh[0])


def test_equal_keys_average_values(ora):
    D, T = 128, 37
    cache = ora.HostCache(1, 1, D, 48, 4, 2, 64)
    rng = np.random.default_rng(2)
    k = np.repeat(rng.standard_normal((1, 1, 1, D)).astype(np.float32), T, axis=2)
    v = rng.standard_normal((1, 1, T, D)).astype(np.float32)
    cache.quantize_append(k, v, [0])
    q = rng.standard_normal((1, 1, D)).astype(np.float32)
    out, _ = cache.decode_attention(q, 1, [T])
    _, vh = _deq(cache, 0, 0, T)
    assert np.allclose(out[0, 0], vh.mean(axis=0), rtol=0, atol=1e-13)


def test_dominant_score_selects_value(ora):
    cache, _, _ = _filled_cache(ora, 1, 1, 64, 20, G=32, seed=3)
    kh, vh = _deq(cache, 0, 0, 20)
    q = (kh[7] / np.linalg.norm(kh[7])).astype(np.float32)[None, None, :]
    out, _ = cache.decode_attention(q, 1, [20], sm_scale=1e4)
    assert np.abs(out[0, 0] - vh[np.argmax(kh @ q[0, 0].astype(np.float64))]).max() < 1e-9


@pytest.mark.parametrize("T", [1, 2, 3, 5])
def test_brute_force_tiny(ora, T):
    D = 64
    cache, _, _ = _filled_cache(ora, 1, 1, D, T, G=32, seed=10 + T)
    q = np.random.default_rng(T).standard_normal((1, 1, D)).astype(np.float32)
    out, _ = cache.decode_attention(q, 1, [T], sm_scale=0.3)
    kh, vh = _deq(cache, 0, 0, T)
    s = []
    for t in range(T):
        acc = 0.0
        for d in range(D):
            acc += float(q[0, 0, d]) * float(kh[t, d])
        s.append(acc * float(np.float32(0.3)))
    m = max(s)
    e = [math.exp(x - m) for x in s]
    tot = sum(e)
    want = [sum(e[t] * float(vh[t, d]) for t in range(T)) / tot for d in range(D)]
    assert np.allclose(out[0, 0], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bk,bv,G", [(4, 2, 64), (8, 4, 32), (2, 4, 128)])
def test_library_softmax_gqa(ora, bk, bv, G):
    B, Hkv, Hq, D, T = 2, 2, 8, 128, 70
    cache, _, _ = _filled_cache(ora, B, Hkv, D, T, bk, bv, G, seed=4)
    q = np.random.default_rng(5).standard_normal((B, Hq, D)).astype(np.float32)
    lens = [70, 33]
    out, _ = cache.decode_attention(q, Hq, lens)
    for b in range(B):
        for hq in range(Hq):
            kh, vh = _deq(cache, b, hq // (Hq // Hkv), lens[b])
            p = softmax(kh @ q[b, hq].astype(np.float64) / math.sqrt(D))
            assert np.allclose(out[b, hq], p @ vh, rtol=0, atol=1e-12)


def test_empty_sequence_and_clamp(ora):
    cache, _, _ = _filled_cache(ora, 2, 1, 64, 32, G=32, seed=6)
    q = np.ones((2, 1, 64), np.float32)
    out, flags = cache.decode_attention(q, 1, [0, 32])
    assert flags == 0 and not out[0].any()
    out2, flags2 = cache.decode_attention(q, 1, [0, 40])      # > capacity 32
    assert flags2 == 2 and np.array_equal(out2, out)
    out3, flags3 = cache.decode_attention(q, 1, [0, 32], max_len=16)
    ref, _ = cache.decode_attention(q, 1, [0, 16])
    assert flags3 == 2 and np.array_equal(out3, ref)


def test_bf16_query_is_widened_exactly(ora):
    import torch
    cache, _, _ = _filled_cache(ora, 1, 2, 128, 40, seed=7)
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    qb, dt = workloads.as_bits(q)
    out_b, _ = cache.decode_attention(qb, 4, [40], q_dtype=dt)
    out_f, _ = cache.decode_attention(q.float().numpy(), 4, [40])
    assert np.array_equal(out_b, out_f)


def test_dense_attention_library(ora):
    rng = np.random.default_rng(8)
    B, Hkv, Hq, D, T = 2, 2, 6, 64, 50
    k = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    lens = [50, 17]
    out = ora.attention_dense(k, v, q, lens)
    for b in range(B):
        for hq in range(Hq):
            h = hq // 3
            kk = k[b, h, :lens[b]].astype(np.float64)
            p = softmax(kk @ q[b, hq].astype(np.float64) / 8.0)
            assert np.allclose(out[b, hq], p @ v[b, h, :lens[b]].astype(np.float64), atol=1e-12)
