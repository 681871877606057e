"""The page's checkable claims, pinned on the oracle (fixtures in golden/).

"Quantize What Counts: More for Keys, Less for Values" (summary page):
  * "Key contributions": K4V2 saves 25% of KV-cache memory against K4V4;
  * "Results", reconstruction error: keys err more than values at equal bits;
  * "Methodology" / "Results": K4V2 beats K2V4 at the same budget.
"""
import json
import os

import numpy as np
import pytest

from kv_cache_mixed_kvq_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_claims.json")


def _claim(cid):
    with open(GOLDEN) as f:
        return {c["id"]: c for c in json.load(f)["claims"]}[cid]


def test_memory_claim_oracle_sizes(ora):
    c = _claim("memory_k4v2_vs_k4v4")
    a = ora.HostCache(1, 8, 128, 4096, 4, 2, 64)
    b = ora.HostCache(1, 8, 128, 4096, 4, 4, 64)
    codes = lambda x: x.k_codes.nbytes + x.v_codes.nbytes
    total = lambda x: codes(x) + x.k_params.nbytes + x.v_params.nbytes
    assert 1 - codes(a) / codes(b) == c["value"]
    assert total(a) / total(b) == pytest.approx(7 / 9, abs=1e-12)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_key_error_exceeds_value_error(ora, bits):
    _claim("key_error_exceeds_value_error")
    w = workloads.WORKLOADS["llama3_8b"]
    k, v = workloads.make_kv(w, 64, seed=11, batch=1)
    cache = ora.HostCache(1, w.kv_heads, 128, 64, bits, bits, 64)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    cache.quantize_append(kb, vb, [0], dtype=dt)
    ek = ev = 0.0
    for h in range(w.kv_heads):
        ek += np.abs(cache.dequant_slot(0, 0, h, 64) - k[0, h].float().numpy()).mean()
        ev += np.abs(cache.dequant_slot(1, 0, h, 64) - v[0, h].float().numpy()).mean()
    assert ek > ev


def test_key_priority_k4v2_beats_k2v4(ora):
    _claim("key_priority_k4v2_beats_k2v4")
    w = workloads.WORKLOADS["qwen_mistral"]
    B, T = 2, 512          # reduced batch/length so the CPU pin stays quick
    k, v = workloads.make_kv(w, T, seed=0, batch=B)
    q = workloads.make_q(w, seed=0, batch=B)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    qb, _ = workloads.as_bits(q)
    ref = ora.attention_dense(kb, vb, qb, [T] * B, kv_dtype=dt, q_dtype=dt)
    errs = {}
    for bk, bv in ((4, 2), (2, 4)):
        cache = ora.HostCache(B, w.kv_heads, 128, T, bk, bv, 64)
        cache.quantize_append(kb, vb, [0] * B, dtype=dt)
        out, _ = cache.decode_attention(qb, w.q_heads, [T] * B, q_dtype=dt)
        errs[(bk, bv)] = (np.linalg.norm(out - ref) / np.linalg.norm(ref), np.abs(out - ref).max())
    assert errs[(4, 2)][0] < errs[(2, 4)][0]
    assert errs[(4, 2)][1] < errs[(2, 4)][1]
