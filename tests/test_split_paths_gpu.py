"""The two ways decode attention finishes a row.

With one split per row (every length fits in one split) each CTA writes its
rows' final output and no workspace is needed; with several, the CTAs write
partial results and the log-sum-exp combine kernel merges them.  Both must
agree with the oracle, under CUDA-graph replay too, and empty sequences must
produce zeros on both paths.
"""
import os

import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, both_quantize, compare_attention

pytestmark = pytest.mark.gpu


def _setup(ora, lens, B=3, Hkv=2, gq=4, D=128, seed=0):
    T = max(lens)
    cap = max((T + 15) // 16 * 16, 16)
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Hkv, max(T, 1), D, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, max(T, 1), D, generator=g).to(torch.bfloat16)
    cache, hc = both_quantize(ora, (B, Hkv, D, cap, 4, 2, 64), k, v, [0] * B)
    q = torch.randn(B, Hkv * gq, D, generator=g).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    ref, _ = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=T)
    return cache, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), T, ref


def _decode(cache, q, lens, T, split):
    old = os.environ.get("KVQ_SPLIT_TOKENS")
    os.environ["KVQ_SPLIT_TOKENS"] = str(split)
    try:
        need = kvq.kvq_decode_workspace_bytes(cache, q.shape[1], T)
        out = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        if old is None:
            del os.environ["KVQ_SPLIT_TOKENS"]
        else:
            os.environ["KVQ_SPLIT_TOKENS"] = old
    return out, need


@pytest.mark.parametrize("split,direct", [(2048, True), (256, False), (64, False)])
def test_direct_and_combined_rows_match_the_oracle(ora, split, direct):
    cache, q, lens, T, ref = _setup(ora, [2048, 700, 65])
    out, need = _decode(cache, q, lens, T, split)
    assert (need == 0) == direct
    compare_attention(out, ref, TOL)


@pytest.mark.parametrize("split", [4096, 256])
def test_empty_sequences_give_zeros_on_both_paths(ora, split):
    cache, q, lens, T, ref = _setup(ora, [0, 640, 0], seed=7)
    out, _ = _decode(cache, q, lens, T, split)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    compare_attention(out, ref, TOL)


def test_graph_replays_give_identical_results(ora):
    cache, q, lens, T, ref = _setup(ora, [1024, 900, 300], seed=5)
    need = kvq.kvq_decode_workspace_bytes(cache, q.shape[1], T)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention(cache, q, lens, T, out=out, workspace=ws)  # loads the kernels
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
