"""Pins of the oracle's key-only rotation (summary page "Quantize What Counts:
More for Keys, Less for Values", "Results", "Integration with rotation":
rotating only the keys of a K4V2 cache comes close to K4V4).

The rotation is the unnormalised Walsh-Hadamard transform H (Sylvester
order) along head_dim: keys are stored as H k, queries become H q / D, and
(H q / D) . (H k) = q . k because H H = D I.
"""
import numpy as np
import pytest
import scipy.linalg

from kv_cache_mixed_kvq_b200 import workloads


@pytest.mark.parametrize("n", [64, 128])
def test_fwht_is_the_sylvester_hadamard_product(ora, n):
    rng = np.random.default_rng(n)
    x = rng.integers(-1000, 1000, size=n).astype(np.float32)  # exact in binary32
    expected = scipy.linalg.hadamard(n).astype(np.float64) @ x.astype(np.float64)
    np.testing.assert_array_equal(ora.fwht(x).astype(np.float64), expected)


@pytest.mark.parametrize("n", [64, 128])
def test_fwht_twice_is_n_times_identity(ora, n):
    for i in (0, 1, n // 2 + 3, n - 1):
        e = np.zeros(n, np.float32)
        e[i] = 1.0
        np.testing.assert_array_equal(ora.fwht(ora.fwht(e)), n * e)


def test_fwht_rounds_in_binary32_butterfly_order(ora):
    # values whose sums round in binary32: the result must equal the
    # butterfly evaluated step by step in binary32 (not an exact dot product)
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(64) * np.exp2(rng.integers(-12, 12, 64))).astype(np.float32)
    y = x.copy()
    h = 1
    while h < 64:
        for i in range(64):
            if i & h == 0:
                a, b = y[i], y[i + h]
                y[i], y[i + h] = np.float32(a + b), np.float32(a - b)
        h *= 2
    np.testing.assert_array_equal(ora.fwht(x), y)


def test_rotated_keys_dequantise_near_the_rotated_row(ora):
    w = workloads.WORKLOADS["llama3_8b"]
    k, v = workloads.make_kv(w, 16, seed=3, batch=1)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    hc = ora.HostCache(1, w.kv_heads, w.head_dim, 16, 8, 4, w.group, rotate_keys=True)
    assert hc.quantize_append(kb, vb, [0], dtype=dt) == 0
    for h in range(w.kv_heads):
        for p in range(16):
            rot = ora.fwht(k[0, h, p].float().numpy())
            deq = hc.dequant_row(0, 0, h, p)
            for g in range(w.head_dim // w.group):
                sl = slice(g * w.group, (g + 1) * w.group)
                span = rot[sl].max() - rot[sl].min()
                # half a level plus the binary16 rounding of scale and zero
                assert np.abs(deq[sl] - rot[sl]).max() <= span / 255 * 0.5 + 2e-3 * (
                    np.abs(rot[sl]).max() + span)
            # values are not rotated
            vdeq = hc.dequant_row(1, 0, h, p)
            assert np.abs(vdeq - v[0, h, p].float().numpy()).max() < 0.5


def test_rotated_decode_matches_dense_attention_at_8_bits(ora):
    # (H q / D) . (H k) = q . k: with 8-bit keys and values the rotated cache
    # must reproduce unquantised attention closely (a missing 1/D, an
    # unrotated query or a transposed transform would not)
    w = workloads.WORKLOADS["llama3_8b"]
    T = 96
    k, v = workloads.make_kv(w, T, seed=5, batch=1)
    q = workloads.make_q(w, seed=5, batch=1)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    qb, _ = workloads.as_bits(q)
    dense = ora.attention_dense(k.float().numpy(), v.float().numpy(), q.float().numpy(), [T])
    hc = ora.HostCache(1, w.kv_heads, w.head_dim, T, 8, 8, w.group, rotate_keys=True)
    hc.quantize_append(kb, vb, [0], dtype=dt)
    out, flags = hc.decode_attention(qb, w.q_heads, [T], q_dtype=dt)
    assert flags == 0
    # measured: mean 3.8e-3, max 4.6e-2 (outlier keys make some heads peaked);
    # the same cache without rotation gives mean 5.8e-3, max 4.9e-2
    err = np.abs(out - dense)
    assert err.mean() < 1e-2 and err.max() < 0.1


def test_key_only_rotation_brings_k4v2_to_k4v4(ora):
    # the page's claim on keys with outlier channels (key norms ~4x values):
    # K4V2 with rotated keys has the attention error of unrotated K4V4
    w = workloads.WORKLOADS["qwen_mistral"]
    T = 512
    err = {}
    for seed in range(2):
        k, v = workloads.make_kv(w, T, seed=seed, batch=1)
        q = workloads.make_q(w, seed=seed, batch=1)
        kb, dt = workloads.as_bits(k)
        vb, _ = workloads.as_bits(v)
        qb, _ = workloads.as_bits(q)
        dense = ora.attention_dense(k.float().numpy(), v.float().numpy(), q.float().numpy(), [T])
        for bits, rot in (((4, 2), False), ((4, 2), True), ((4, 4), False)):
            hc = ora.HostCache(1, w.kv_heads, w.head_dim, T, bits[0], bits[1], w.group,
                               rotate_keys=rot)
            hc.quantize_append(kb, vb, [0], dtype=dt)
            out, _ = hc.decode_attention(qb, w.q_heads, [T], q_dtype=dt)
            err.setdefault((bits, rot), []).append(np.abs(out - dense).mean())
    e42, e42r, e44 = (float(np.mean(err[k])) for k in (((4, 2), False), ((4, 2), True),
                                                      ((4, 4), False)))
    assert e42r < 0.85 * e42
    assert e42r < 1.15 * e44
