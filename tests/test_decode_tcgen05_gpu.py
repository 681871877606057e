"""The tensor-memory (tcgen05) decode kernel, selected with
KVQ_DECODE_KERNEL=tcgen05, against the binary64 oracle: every bit pair, the
key/value group pairs, 4 and 8 heads per CTA, partial tiles, several splits
and rows of length 1.  It computes the same attention as the default
register-fragment kernel; both are checked against the same bound."""
import os

import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, compare_attention

pytestmark = pytest.mark.gpu


@pytest.fixture
def tcgen05_kernel(monkeypatch):
    monkeypatch.setenv("KVQ_DECODE_KERNEL", "tcgen05")
    yield


@pytest.mark.parametrize("B,Hkv,Hq,T,bits,G,Gv,lens", [
    (1, 1, 4, 128, (4, 2), 64, 0, [128]),
    (1, 1, 4, 200, (4, 2), 64, 0, [200]),
    (2, 2, 8, 700, (4, 2), 64, 0, [700, 333]),
    (2, 8, 32, 3000, (4, 2), 64, 0, [3000, 1]),
    (1, 4, 28, 1500, (2, 4), 64, 0, [1500]),
    (1, 8, 32, 2048, (8, 4), 64, 0, [2048]),
    (1, 8, 32, 2048, (8, 8), 32, 0, [2048]),
    (1, 8, 32, 2048, (2, 2), 128, 0, [2048]),
    (1, 8, 32, 1024, (4, 2), 32, 64, [1024]),
    (2, 2, 16, 1024, (4, 4), 64, 0, [1024, 517]),
])
def test_tcgen05_kernel_matches_oracle(ora, tcgen05_kernel, B, Hkv, Hq, T, bits, G, Gv, lens):
    g = torch.Generator().manual_seed(B * 1000 + T)
    cap = (T + 15) // 16 * 16
    cache = kvq.KVCache.allocate(B, Hkv, 128, cap, bits[0], bits[1], G, group_v=Gv)
    k = (torch.randn(B, Hkv, T, 128, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, 128, generator=g).to(torch.bfloat16)
    kvq.kvq_quantize_append(cache, k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16).cuda()
    L = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = kvq.kvq_decode_attention(cache, q, L, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error_flags() == 0
    hc = ora.HostCache(B, Hkv, 128, cap, bits[0], bits[1], G, group_v=Gv or None)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    hc.quantize_append(kb, vb, [0] * B, dtype=dt)
    qb, qd = workloads.as_bits(q)
    ref, _ = hc.decode_attention(qb, Hq, lens, q_dtype=qd, max_len=T)
    compare_attention(out, ref, TOL)


def test_tcgen05_kernel_flags_a_timeout_and_recovers(tcgen05_kernel):
    B, Hkv, Hq, D, T = 2, 8, 32, 128, 2048
    g = torch.Generator().manual_seed(3)
    cache = kvq.KVCache.allocate(B, Hkv, D, T, 4, 2, 64)
    k = (torch.randn(B, Hkv, T, D, generator=g) * 2).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16).cuda()
    kvq.kvq_quantize_append(cache, k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16).cuda()
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    ref = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0
    kvq.kvq_debug_inject_wait_timeout(1, wait_limit_ns=1_000_000)
    kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() & kvq.KVQ_DEVERR_TIMEOUT
    again = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0
    assert torch.equal(again, ref)
