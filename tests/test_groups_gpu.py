"""GPU parity of separate key and value group sizes (cache descriptor
`group_v`): keys in groups of Gk, values in coarser groups of Gv.  The packed
cache must be bit-identical to the oracle's for every bit pair, head_dim,
input type and append alignment, and decode attention must match the
binary64 oracle within 2e-3 for every query variant; combinations with finer
value groups than key groups are refused."""
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, append, assert_same_cache, compare_attention

pytestmark = pytest.mark.gpu


def _inputs(B, Hkv, T, D, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    centre = torch.randn(Hkv, 1, D, generator=g) * 2
    mult = 1 + 9 * (torch.rand(Hkv, 1, D, generator=g) < 0.03)
    k = ((centre + torch.randn(B, Hkv, T, D, generator=g)) * mult).to(dtype)
    v = torch.randn(B, Hkv, T, D, generator=g).to(dtype)
    return k, v


def _pair(ora, B, Hkv, D, cap, bk, bv, gk, gv, rotate=False):
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, bk, bv, gk, group_v=gv, rotate_keys=rotate)
    hc = ora.HostCache(B, Hkv, D, cap, bk, bv, gk, group_v=gv, rotate_keys=rotate)
    return cache, hc


COMBOS = [(128, 32, 64), (128, 32, 128), (128, 64, 128), (64, 32, 64)]


@pytest.mark.parametrize("D,gk,gv", COMBOS)
@pytest.mark.parametrize("bk,bv", [(4, 2), (8, 4), (2, 4), (8, 8)])
def test_cache_bit_exact(ora, D, gk, gv, bk, bv):
    k, v = _inputs(2, 2, 40, D, seed=gk + gv + bk)
    cache, hc = _pair(ora, 2, 2, D, 64, bk, bv, gk, gv)
    fo, fg = append(ora, cache, hc, k, v, [0, 9])
    assert fo == 0 and fg == 0
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_cache_bit_exact_input_types_and_appends(ora, dtype):
    cache, hc = _pair(ora, 2, 2, 128, 80, 4, 2, 32, 128)
    for (pos, n), seed in zip([((0, 3), 17), ((17, 20), 30)], range(2)):
        k, v = _inputs(2, 2, n, 128, seed=seed + 50, dtype=dtype)
        append(ora, cache, hc, k, v, list(pos))
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("D,gk,gv", COMBOS)
@pytest.mark.parametrize("gq,q_dtype", [(4, torch.bfloat16), (7, torch.bfloat16),
                                        (8, torch.float32), (2, torch.float16)])
def test_decode_matches_oracle(ora, D, gk, gv, gq, q_dtype):
    B, Hkv, lens = 2, 2, [333, 70]
    T = max(lens)
    cap = (T + 15) // 16 * 16
    k, v = _inputs(B, Hkv, T, D, seed=gq + gk)
    cache, hc = _pair(ora, B, Hkv, D, cap, 4, 2, gk, gv)
    append(ora, cache, hc, k, v, [0] * B)
    q = torch.randn(B, Hkv * gq, D, generator=torch.Generator().manual_seed(gq)).to(q_dtype)
    qb, qdt = workloads.as_bits(q)
    ref, _ = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=T)
    out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor(lens, dtype=torch.int32,
                                                                 device="cuda"),
                                   T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    compare_attention(out, ref, TOL)


def test_rotated_keys_with_separate_groups(ora):
    B, Hkv, gq, D, lens = 1, 2, 4, 128, [257]
    k, v = _inputs(B, Hkv, 257, D, seed=99)
    cache, hc = _pair(ora, B, Hkv, D, 272, 4, 2, 32, 128, rotate=True)
    append(ora, cache, hc, k, v, [0])
    assert_same_cache(cache, hc)
    q = torch.randn(B, Hkv * gq, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    ref, _ = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=257)
    out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor(lens, dtype=torch.int32,
                                                                 device="cuda"),
                                   257, out_dtype=torch.float32)
    torch.cuda.synchronize()
    compare_attention(out, ref, TOL)


def test_finer_value_groups_are_refused():
    cache = kvq.KVCache.allocate(1, 1, 128, 64, 4, 2, 64, group_v=32)
    k = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_quantize_append(cache, k, k, torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
