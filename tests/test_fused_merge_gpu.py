"""The in-kernel split merge of decode attention.

Rows with one split are written directly by their CTA; rows with 2..16
splits are merged by the last CTA of each (batch row, kv head) to finish,
counted on epoch-tagged arrival counters in the workspace; longer rows go
through the separate combine kernel.  These tests check that all three
paths agree with the oracle, that the counters need no initialisation
(garbage workspace) and reset themselves (CUDA-graph replays of one call),
and that empty sequences produce zeros.
"""
import os

import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, both_quantize, compare_attention

pytestmark = pytest.mark.gpu


def _setup(ora, lens, B=3, Hkv=2, gq=4, D=128, seed=0):
    T = max(lens)
    cap = (T + 15) // 16 * 16
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Hkv, max(T, 1), D, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, max(T, 1), D, generator=g).to(torch.bfloat16)
    cache, hc = both_quantize(ora, (B, Hkv, D, max(cap, 16), 4, 2, 64), k, v, [0] * B)
    q = torch.randn(B, Hkv * gq, D, generator=g).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    ref, _ = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=T)
    return cache, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), T, ref


def _decode(cache, q, lens, T, split=None, workspace=None):
    old = os.environ.get("KVQ_SPLIT_TOKENS")
    if split:
        os.environ["KVQ_SPLIT_TOKENS"] = str(split)
    try:
        out = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32,
                                       workspace=workspace)
        torch.cuda.synchronize()
    finally:
        if split:
            if old is None:
                del os.environ["KVQ_SPLIT_TOKENS"]
            else:
                os.environ["KVQ_SPLIT_TOKENS"] = old
    return out


@pytest.mark.parametrize("split", [2048, 256, 128, 64])  # 1, 8, 16 and 32 splits of the longest row
def test_direct_fused_and_combine_paths_match_the_oracle(ora, split):
    cache, q, lens, T, ref = _setup(ora, [2048, 700, 65])
    out = _decode(cache, q, lens, T, split=split)
    compare_attention(out, ref, TOL)


def test_counters_need_no_initialisation(ora):
    cache, q, lens, T, ref = _setup(ora, [1500, 1500, 33], seed=3)
    old = os.environ.get("KVQ_SPLIT_TOKENS")
    os.environ["KVQ_SPLIT_TOKENS"] = "256"  # 6 splits: merged in the kernel
    try:
        need = kvq.kvq_decode_workspace_bytes(cache, q.shape[1], T)
    finally:
        if old is None:
            del os.environ["KVQ_SPLIT_TOKENS"]
        else:
            os.environ["KVQ_SPLIT_TOKENS"] = old
    for fill in (0xFF, 0x00, 0x5A):
        ws = torch.full((need,), fill, dtype=torch.uint8, device="cuda")
        out = _decode(cache, q, lens, T, split=256, workspace=ws)
        compare_attention(out, ref, TOL)


def test_graph_replays_reset_the_counters(ora):
    cache, q, lens, T, ref = _setup(ora, [1024, 900, 300], seed=5)
    need = kvq.kvq_decode_workspace_bytes(cache, q.shape[1], T)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention(cache, q, lens, T, out=out, workspace=ws)  # warm-up, loads kernels
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kvq.kvq_decode_attention(cache, q, lens, T, out=out, workspace=ws)
    results = []
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        results.append(out.clone())
    for r in results:
        compare_attention(r, ref, TOL)
        assert torch.equal(r, results[0])
    assert kvq.kvq_device_error_flags() == 0


def test_empty_sequences_give_zeros_on_every_path(ora):
    for split in (4096, 256):
        cache, q, lens, T, ref = _setup(ora, [0, 640, 0], seed=7)
        out = _decode(cache, q, lens, T, split=split)
        assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
        compare_attention(out, ref, TOL)
