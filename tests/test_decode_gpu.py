"""GPU decode attention vs the binary64 oracle on the oracle's own cache.

The GPU quantizes and attends on its side, the oracle on its side, from the
same inputs; outputs must agree within 2e-3 max-abs (plus half a bf16 ulp for
bf16 outputs).  Covers every bit-width pair, both head dims, all groups,
grouped-query ratios 1..16, ragged and tiny lengths, split counts, query and
output types, empty sequences and length clamping.
"""
import os

import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, both_quantize, compare_attention

pytestmark = pytest.mark.gpu


def _kvq_inputs(B, Hkv, T, D, seed, dtype=torch.bfloat16, outliers=True):
    g = torch.Generator().manual_seed(seed)
    centre = torch.randn(Hkv, 1, D, generator=g) * 2
    mult = 1 + 9 * (torch.rand(Hkv, 1, D, generator=g) < 0.03) if outliers else 1
    k = ((centre + torch.randn(B, Hkv, T, D, generator=g)) * mult).to(dtype)
    v = torch.randn(B, Hkv, T, D, generator=g).to(dtype)
    return k, v


def _run(ora, B, Hkv, Hq, D, bk, bv, G, lens, q_dtype=torch.bfloat16, out_dtype=torch.float32,
         seed=0, sm_scale=0.0, kv_dtype=torch.bfloat16, split_tokens=None, max_len=None):
    T = max(max(lens), 1)
    cap = (T + 15) // 16 * 16
    k, v = _kvq_inputs(B, Hkv, T, D, seed, kv_dtype)
    cache, hc = both_quantize(ora, (B, Hkv, D, cap, bk, bv, G), k, v, [0] * B)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(seed + 1)).to(q_dtype)
    qb, qdt = workloads.as_bits(q)
    max_len = T if max_len is None else max_len
    ref, _ = hc.decode_attention(qb, Hq, lens, sm_scale=sm_scale, q_dtype=qdt, max_len=max_len)
    old = os.environ.get("KVQ_SPLIT_TOKENS")
    if split_tokens:
        os.environ["KVQ_SPLIT_TOKENS"] = str(split_tokens)
    try:
        out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor(lens, dtype=torch.int32,
                                                                     device="cuda"),
                                       max_len, sm_scale=sm_scale, out_dtype=out_dtype)
        torch.cuda.synchronize()
    finally:
        if split_tokens:
            if old is None:
                del os.environ["KVQ_SPLIT_TOKENS"]
            else:
                os.environ["KVQ_SPLIT_TOKENS"] = old
    return out, ref


BITS = [(bk, bv) for bk in (2, 4, 8) for bv in (2, 4, 8)]


@pytest.mark.parametrize("bk,bv", BITS)
@pytest.mark.parametrize("D,G", [(128, 64), (128, 32), (128, 128), (64, 32), (64, 64)])
def test_bits_dims_groups(ora, bk, bv, D, G):
    out, ref = _run(ora, 2, 2, 8, D, bk, bv, G, [77, 130], seed=bk * 10 + bv + D + G)
    compare_attention(out, ref)


@pytest.mark.parametrize("gq", [1, 2, 3, 4, 5, 7, 8, 12, 16])
@pytest.mark.parametrize("q_dtype", [torch.bfloat16, torch.float32, torch.float16])
def test_gqa_ratios_and_query_types(ora, gq, q_dtype):
    out, ref = _run(ora, 2, 2, 2 * gq, 128, 4, 2, 64, [100, 37], q_dtype=q_dtype, seed=gq)
    compare_attention(out, ref)


@pytest.mark.parametrize("lens", [[1], [2], [15], [16], [17], [31], [33], [63], [64], [65],
                                  [257], [1, 2, 3, 200], [0, 50], [0, 0]])
def test_lengths_and_tails(ora, lens):
    out, ref = _run(ora, len(lens), 1, 4, 128, 4, 2, 64, lens, seed=sum(lens))
    compare_attention(out, ref)
    for b, n in enumerate(lens):
        if n == 0:
            assert not out[b].any()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_output_types(ora, out_dtype):
    out, ref = _run(ora, 2, 2, 8, 128, 4, 2, 64, [300, 100], out_dtype=out_dtype, seed=5)
    compare_attention(out, ref)


def test_fp32_tiny_config(ora):
    # single head, head_dim 64, 256 tokens, fp32 inputs, K4V2 group 32
    w = workloads.WORKLOADS["tiny"]
    k, v = workloads.make_kv(w, w.context, seed=0)
    q = workloads.make_q(w, seed=0)
    cache, hc = both_quantize(ora, (1, 1, 64, 256, 4, 2, 32), k, v, [0])
    ref, _ = hc.decode_attention(q.numpy(), 1, [256])
    for out_dtype in (torch.float32, torch.bfloat16):
        out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor([256], dtype=torch.int32,
                                                                     device="cuda"), 256,
                                       out_dtype=out_dtype)
        err = compare_attention(out, ref)
        if out_dtype == torch.float32:
            assert err < 1e-4


def test_split_count_invariance(ora):
    outs = []
    for st in (64, 128, 256, 1024, 4096):
        out, ref = _run(ora, 2, 2, 8, 128, 4, 2, 64, [1000, 613], seed=11, split_tokens=st)
        compare_attention(out, ref)
        outs.append(out.cpu().numpy())
    # Splits change the order of the sums and the softmax reference maxima;
    # the tensor cores truncate products of binary16 subnormal operands to
    # about 2^-19.6 of the sum of |terms| per instruction (measured), so the
    # outputs of different split counts agree to ~1e-4, far inside the 2e-3
    # bar, while a wrong log-sum-exp weight would move them by O(0.1).
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2e-4


def test_sm_scale_and_peaked_softmax(ora):
    out, ref = _run(ora, 1, 1, 4, 128, 4, 2, 64, [500], sm_scale=2.0, seed=13)
    compare_attention(out, ref)
    out, ref = _run(ora, 1, 1, 4, 128, 8, 4, 64, [500], sm_scale=0.01, seed=14)
    compare_attention(out, ref)


def test_length_clamping_flags(ora):
    out, ref = _run(ora, 2, 1, 2, 64, 4, 2, 32, [40, 40], max_len=32, seed=15)
    compare_attention(out, ref)
    assert kvq.kvq_device_error_flags() & kvq.KVQ_DEVERR_SEQ_LEN
    # the single-value form reads the same word, and reading clears it
    _run(ora, 2, 1, 2, 64, 4, 2, 32, [40, 40], max_len=32, seed=15)
    assert kvq.kvq_last_device_error() == kvq.KVQ_DEVERR_SEQ_LEN
    assert kvq.kvq_last_device_error() == 0


def test_workspace_too_small_is_rejected():
    # 4096 tokens for one (batch row, kv head): several splits, so partial
    # results (and arrival counters) need a workspace
    cache = kvq.KVCache.allocate(1, 1, 128, 4096, 4, 2, 64)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([4096], dtype=torch.int32, device="cuda")
    assert kvq.kvq_decode_split_tokens(cache, 4, 4096) < 4096
    need = kvq.kvq_decode_workspace_bytes(cache, 4, 4096)
    assert need > 0
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention(cache, q, lens, 4096, workspace=ws)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE


def test_single_split_needs_no_workspace():
    # one split per row: each CTA writes its rows' final output directly
    cache = kvq.KVCache.allocate(1, 1, 128, 64, 4, 2, 64)
    assert kvq.kvq_decode_split_tokens(cache, 4, 64) == 64
    assert kvq.kvq_decode_workspace_bytes(cache, 4, 64) == 0
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([64], dtype=torch.int32, device="cuda")
    out = kvq.kvq_decode_attention(cache, q, lens, 64)  # no workspace
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("lens", [[1000, 613, 77, 0, 2048, 129], [4096], [300, 0, 0, 5000]])
def test_balanced_schedule(ora, lens, monkeypatch):
    # the opt-in one-wave schedule: spans cross unit and row boundaries
    monkeypatch.setenv("KVQ_DECODE_SCHEDULE", "balanced")
    out, ref = _run(ora, len(lens), 2, 8, 128, 4, 2, 64, lens, seed=21 + len(lens))
    compare_attention(out, ref)
    for b, n in enumerate(lens):
        if n == 0:
            assert not out[b].any()


@pytest.mark.parametrize("q_dtype,offset", [(torch.bfloat16, 1), (torch.float32, 1),
                                            (torch.float16, 4)])
def test_unaligned_query_is_rejected(q_dtype, offset):
    # the query rows are bulk-copied: a query not on 16 bytes is an invalid
    # argument, and nothing is launched
    cache = kvq.KVCache.allocate(1, 1, 128, 64, 4, 2, 64)
    buf = torch.zeros(4 * 128 + offset, dtype=q_dtype, device="cuda")
    q = buf[offset:].view(1, 4, 128)
    assert q.data_ptr() % 16 != 0
    lens = torch.tensor([64], dtype=torch.int32, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention(cache, q, lens, 64)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
