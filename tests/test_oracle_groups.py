"""Pins of separate key and value group sizes in the oracle (summary page
"Quantize What Counts: More for Keys, Less for Values", "Results",
"Group-size sensitivity": finer groups (32) help the keys, coarser ones (64
or 128) are enough for the values).  Keys use groups of Gk elements, values
groups of Gv, each array's (scale, zero) pairs indexed by its own group count.
"""
import numpy as np
import pytest

from kv_cache_mixed_kvq_b200 import workloads


def _cache(ora, w, T, bits, gk, gv, seed=0):
    k, v = workloads.make_kv(w, T, seed=seed, batch=1)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    hc = ora.HostCache(1, w.kv_heads, w.head_dim, T, bits[0], bits[1], gk, group_v=gv)
    assert hc.quantize_append(kb, vb, [0], dtype=dt) == 0
    return hc, k, v


def test_equal_groups_match_the_single_group_cache(ora):
    w = workloads.WORKLOADS["llama3_8b"]
    a, _, _ = _cache(ora, w, 32, (4, 2), 64, 64)
    b, _, _ = _cache(ora, w, 32, (4, 2), 64, None)
    for x, y in ((a.k_codes, b.k_codes), (a.v_codes, b.v_codes), (a.k_params, b.k_params),
                 (a.v_params, b.v_params)):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("gk,gv", [(32, 128), (32, 64), (64, 128)])
def test_each_array_uses_its_own_groups(ora, gk, gv):
    w = workloads.WORKLOADS["llama3_8b"]
    T = 16
    hc, k, v = _cache(ora, w, T, (8, 8), gk, gv, seed=4)
    assert hc.k_params.size == w.kv_heads * T * (w.head_dim // gk) * 2
    assert hc.v_params.size == w.kv_heads * T * (w.head_dim // gv) * 2
    for which, x, g in ((0, k, gk), (1, v, gv)):
        for h in range(w.kv_heads):
            for p in range(T):
                row = x[0, h, p].float().numpy()
                deq = hc.dequant_row(which, 0, h, p)
                for j in range(w.head_dim // g):
                    sl = slice(j * g, (j + 1) * g)
                    span = row[sl].max() - row[sl].min()
                    # half an 8-bit level plus the binary16 rounding of scale and zero
                    assert np.abs(deq[sl] - row[sl]).max() <= span / 255 * 0.5 + 2e-3 * (
                        np.abs(row[sl]).max() + span)


def test_key_groups_matter_more_than_value_groups(ora):
    # Qwen/Mistral-shaped heads with outlier keys, K4V2, mean |error| of the
    # attention output against unquantised binary64 attention (measured:
    # (64,64) 0.098, (32,64) 0.081, (64,128) 0.104, (128,64) 0.143)
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
        for gk, gv in ((64, 64), (32, 64), (64, 128), (128, 64)):
            hc = ora.HostCache(1, w.kv_heads, w.head_dim, T, 4, 2, gk, group_v=gv)
            hc.quantize_append(kb, vb, [0], dtype=dt)
            out, _ = hc.decode_attention(qb, w.q_heads, [T], q_dtype=dt)
            err.setdefault((gk, gv), []).append(np.abs(out - dense).mean())
    e = {key: float(np.mean(val)) for key, val in err.items()}
    assert e[(32, 64)] < 0.9 * e[(64, 64)]      # finer key groups help
    assert e[(64, 128)] < 1.15 * e[(64, 64)]    # coarser value groups cost little
    assert e[(128, 64)] > 1.3 * e[(64, 128)]    # key granularity matters more
