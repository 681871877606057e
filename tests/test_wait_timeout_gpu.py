"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait of the decode kernel's copy pipeline is bounded.  The test knob
kvq_debug_inject_wait_timeout() makes one of the first two pipeline stages of
the next decode launch expect more bytes on its mbarrier than its copies
bring, and shortens the wait limit to one millisecond.  The wait on that stage then runs
out: the kernel must flag KVQ_DEVERR_TIMEOUT, drain its other copies and
return (no hang, no fault), and the context must stay usable: the next
normal call on the same cache reproduces a fresh call bit for bit.
"""
import time

import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq

pytestmark = pytest.mark.gpu


def _cache(B, Hkv, D, T, seed):
    g = torch.Generator().manual_seed(seed)
    cache = kvq.KVCache.allocate(B, Hkv, D, T, 4, 2, 64)
    k = (torch.randn(B, Hkv, T, D, generator=g) * 2).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16).cuda()
    kvq.kvq_quantize_append(cache, k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    return cache


@pytest.mark.parametrize("drop_stage", [0, 1])
def test_wait_runs_out_flags_timeout_and_recovers(drop_stage):
    B, Hkv, Hq, D, T = 2, 8, 32, 128, 2048
    cache = _cache(B, Hkv, D, T, seed=3)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(4)).to(
        torch.bfloat16).cuda()
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    ref = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0

    kvq.kvq_debug_inject_wait_timeout(drop_stage, wait_limit_ns=1_000_000)
    t0 = time.perf_counter()
    kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    flags = kvq.kvq_last_device_error()
    assert flags & kvq.KVQ_DEVERR_TIMEOUT, f"flags {flags}"
    assert elapsed < 0.5  # two waits of 1 ms at most, not the default 1 s

    # the knob is one-shot: the next call is normal and equals a fresh one
    again = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0
    assert torch.equal(again, ref)


def test_knob_rejects_out_of_range_limits_and_disarms():
    with pytest.raises(kvq.KvqError):
        kvq.kvq_debug_inject_wait_timeout(0, wait_limit_ns=10)
    kvq.kvq_debug_inject_wait_timeout(1, wait_limit_ns=1_000_000)
    kvq.kvq_debug_inject_wait_timeout(-1)  # disarmed: the next call is normal
    cache = _cache(1, 8, 128, 512, seed=5)
    q = torch.randn(1, 32, 128, generator=torch.Generator().manual_seed(6)).to(
        torch.bfloat16).cuda()
    lens = torch.full((1,), 512, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attention(cache, q, lens, 512)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0


@pytest.mark.parametrize("drop_stage", [0, 1])
def test_wait_runs_out_under_the_balanced_schedule(drop_stage, monkeypatch):
    # one-wave schedule: the first CTA's range crosses a unit boundary (row
    # 0's units have 3 stages, a CTA takes 4), so when its wait runs out the
    # next span's query rows and stages may already be in flight; they are
    # waited for before the CTA ends
    monkeypatch.setenv("KVQ_DECODE_SCHEDULE", "balanced")
    B, Hkv, Hq, D, T = 2, 8, 32, 128, 2048
    cache = _cache(B, Hkv, D, T, seed=7)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(8)).to(
        torch.bfloat16).cuda()
    lens = torch.tensor([300, T], dtype=torch.int32, device="cuda")
    ref = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0

    kvq.kvq_debug_inject_wait_timeout(drop_stage, wait_limit_ns=1_000_000)
    t0 = time.perf_counter()
    kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    flags = kvq.kvq_last_device_error()
    assert flags & kvq.KVQ_DEVERR_TIMEOUT, f"flags {flags}"
    assert elapsed < 0.5

    again = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_error() == 0
    assert torch.equal(again, ref)
