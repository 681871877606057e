"""GPU parity of the key-only rotation (KVQ_FLAG_ROTATE_KEYS) against the
oracle: keys stored as H k must be bit-identical (codes, scales, zeros) for
every bit width, head_dim, group, input type and append alignment, and
decode attention over a rotated cache (the query rotated to H q / D in the
kernel) must match the binary64 oracle within 2e-3."""
import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, append, assert_same_cache, compare_attention

pytestmark = pytest.mark.gpu


def _inputs(B, Hkv, T, D, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    centre = torch.randn(Hkv, 1, D, generator=g) * 2
    mult = 1 + 9 * (torch.rand(Hkv, 1, D, generator=g) < 0.03)
    k = ((centre + torch.randn(B, Hkv, T, D, generator=g)) * mult).to(dtype)
    v = torch.randn(B, Hkv, T, D, generator=g).to(dtype)
    return k, v


def _pair(ora, B, Hkv, D, cap, bk, bv, G):
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, bk, bv, G, rotate_keys=True)
    hc = ora.HostCache(B, Hkv, D, cap, bk, bv, G, rotate_keys=True)
    return cache, hc


SHAPES = [(128, 4, 2, 64), (128, 8, 4, 64), (128, 2, 4, 64), (128, 4, 2, 32), (128, 2, 2, 128),
          (128, 8, 8, 32), (64, 4, 2, 32), (64, 2, 8, 64), (64, 8, 2, 64)]


@pytest.mark.parametrize("D,bk,bv,G", SHAPES)
def test_rotated_cache_bit_exact(ora, D, bk, bv, G):
    k, v = _inputs(2, 2, 48, D, seed=D + bk * 10 + bv, dtype=torch.bfloat16)
    cache, hc = _pair(ora, 2, 2, D, 64, bk, bv, G)
    fo, fg = append(ora, cache, hc, k, v, [0, 16])
    assert fo == 0 and fg == 0
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_rotated_cache_input_types_and_ragged_appends(ora, dtype):
    cache, hc = _pair(ora, 2, 3, 128, 96, 4, 2, 64)
    for (pos, n), seed in zip([((0, 5), 7), ((7, 12), 9), ((19, 33), 3)], range(3)):
        k, v = _inputs(2, 3, n, 128, seed=seed + 40, dtype=dtype)
        append(ora, cache, hc, k, v, list(pos))
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("D,bk,bv,G,gq,q_dtype", [
    (128, 4, 2, 64, 4, torch.bfloat16),
    (128, 4, 2, 64, 7, torch.bfloat16),
    (128, 8, 4, 64, 4, torch.float32),
    (128, 2, 4, 32, 8, torch.float16),
    (64, 4, 2, 32, 2, torch.bfloat16),
    (128, 4, 4, 128, 1, torch.float32),
])
def test_rotated_decode_matches_oracle(ora, D, bk, bv, G, gq, q_dtype):
    B, Hkv = 2, 2
    lens = [300, 77]
    T = max(lens)
    cap = (T + 15) // 16 * 16
    k, v = _inputs(B, Hkv, T, D, seed=gq * 7 + bk, dtype=torch.bfloat16)
    cache, hc = _pair(ora, B, Hkv, D, cap, bk, bv, G)
    append(ora, cache, hc, k, v, [0] * B)
    assert_same_cache(cache, hc)
    q = torch.randn(B, Hkv * gq, D, generator=torch.Generator().manual_seed(11)).to(q_dtype)
    qb, qdt = workloads.as_bits(q)
    ref, flags = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=T)
    assert flags == 0
    out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor(lens, dtype=torch.int32,
                                                                 device="cuda"),
                                   T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    compare_attention(out, ref, TOL)


def test_key_rotation_on_gpu_brings_k4v2_to_k4v4(ora):
    # the page's claim, on the GPU path (Qwen/Mistral-shaped heads, outlier keys)
    w = workloads.WORKLOADS["qwen_mistral"]
    T = 512
    k, v = workloads.make_kv(w, T, seed=2, batch=1)
    q = workloads.make_q(w, seed=2, batch=1)
    dense = ora.attention_dense(k.float().numpy(), v.float().numpy(), q.float().numpy(), [T])
    err = {}
    for bits, rot in (((4, 2), False), ((4, 2), True), ((4, 4), False)):
        cache = kvq.KVCache.allocate(1, w.kv_heads, w.head_dim, T, bits[0], bits[1], w.group,
                                     rotate_keys=rot)
        kvq.kvq_quantize_append(cache, k.cuda(), v.cuda(), torch.zeros(1, dtype=torch.int32,
                                                                        device="cuda"))
        out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor([T], dtype=torch.int32,
                                                                     device="cuda"),
                                       T, out_dtype=torch.float32)
        err[(bits, rot)] = float(np.abs(out.cpu().numpy() - dense).mean())
    print("mean |error| vs unquantised:", err)
    assert err[((4, 2), True)] < 0.85 * err[((4, 2), False)]
    assert err[((4, 2), True)] < 1.2 * err[((4, 4), False)]
