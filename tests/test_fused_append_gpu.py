"""GPU parity of the fused append + decode call (kvq_append_decode_attention)
against the oracle's definition (append at seq_lens - n_new, then decode):
the cache must be bit-identical, attention within 2e-3 of the binary64
oracle, and both identical, bit for bit, to the two separate GPU calls.
Covered: new tokens crossing split boundaries, several head-group CTAs of one
kv head writing the same rows, every input type, head_dim 64, other bit
pairs and groups, rotated keys, the paged layout, and the rows that append
nothing (too short: flagged; clamped)."""
import os

import numpy as np
import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, assert_same_cache, compare_attention

pytestmark = pytest.mark.gpu


def _inputs(B, Hkv, T, D, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    centre = torch.randn(Hkv, 1, D, generator=g) * 2
    mult = 1 + 9 * (torch.rand(Hkv, 1, D, generator=g) < 0.03)
    k = ((centre + torch.randn(B, Hkv, T, D, generator=g)) * mult).to(dtype)
    v = torch.randn(B, Hkv, T, D, generator=g).to(dtype)
    return k, v


class _Split:
    """Split override (tokens), or "balanced" for the opt-in one-wave schedule."""

    def __init__(self, n):
        self.n = n

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in ("KVQ_SPLIT_TOKENS", "KVQ_DECODE_SCHEDULE")}
        if self.n == "balanced":
            os.environ["KVQ_DECODE_SCHEDULE"] = "balanced"
        elif self.n:
            os.environ["KVQ_SPLIT_TOKENS"] = str(self.n)

    def __exit__(self, *exc):
        for k, v in self.old.items():
            os.environ.pop(k, None)
            if v is not None:
                os.environ[k] = v


def _gpu_row(cache, b):
    """KVCache over batch row b (slot layout: views of its slices; paged: the
    pool with row b's block table)."""
    if cache.page_size:
        return kvq.KVCache(1, cache.kv_heads, cache.head_dim, cache.capacity, cache.bits_k,
                           cache.bits_v, cache.group, cache.k_codes, cache.v_codes,
                           cache.k_params, cache.v_params, rotate_keys=cache.rotate_keys,
                           group_v=cache.group_v, page_size=cache.page_size,
                           num_pages=cache.num_pages,
                           block_table=cache.block_table[b:b + 1].contiguous())
    ts = [cache.k_codes, cache.v_codes, cache.k_params, cache.v_params]
    per = [t.numel() // cache.batch for t in ts]
    return kvq.KVCache(1, cache.kv_heads, cache.head_dim, cache.capacity, cache.bits_k,
                       cache.bits_v, cache.group, *[t[b * n:(b + 1) * n] for t, n in zip(ts, per)],
                       rotate_keys=cache.rotate_keys, group_v=cache.group_v)


def _ora_row(ora, hc, b):
    if isinstance(hc, ora.PagedHostCache):
        D, bk, bv, g, rot, gv = hc.shape
        r = ora.PagedHostCache(1, hc.Hkv, D, hc.cap, bk, bv, g, hc.P, hc.num_pages,
                               hc.block_table[b:b + 1], rotate_keys=rot, group_v=gv)
        r.pool = hc.pool
        return r
    r = ora.HostCache(1, hc.Hkv, hc.D, hc.cap, hc.bits_k, hc.bits_v, hc.group,
                      rotate_keys=hc.rotate_keys, group_v=hc.group_v)
    for name in ("k_codes", "v_codes", "k_params", "v_params"):
        a = getattr(hc, name)
        n = a.size // hc.B
        setattr(r, name, a[b * n:(b + 1) * n])
    return r


def _prefill(ora, cache, hc, prefix, D, seed, dtype):
    """Rows b = 0.. get positions [0, prefix[b]) on both sides."""
    for b, n in enumerate(prefix):
        if n == 0:
            continue
        k, v = _inputs(1, cache.kv_heads, n, D, seed=seed + b, dtype=dtype)
        kb, dt = workloads.as_bits(k)
        vb, _ = workloads.as_bits(v)
        assert _ora_row(ora, hc, b).quantize_append(kb, vb, [0], dtype=dt) == 0
        kvq.kvq_quantize_append(_gpu_row(cache, b), k.cuda(), v.cuda(),
                                torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert kvq.kvq_device_error_flags() == 0


def _make(ora, B, Hkv, D, cap, bk, bv, G, gv=0, rotate=False, page_size=0, lens=None):
    paged = {}
    if page_size:
        table, num_pages = workloads.make_block_table(lens, cap, page_size, seed=3, spare=2)
        paged = dict(page_size=page_size, num_pages=num_pages,
                     block_table=torch.from_numpy(table))
        hc = ora.PagedHostCache(B, Hkv, D, cap, bk, bv, G, page_size, num_pages, table,
                                rotate_keys=rotate, group_v=gv or None)
    else:
        hc = ora.HostCache(B, Hkv, D, cap, bk, bv, G, rotate_keys=rotate, group_v=gv or None)
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, bk, bv, G, group_v=gv, rotate_keys=rotate,
                                 **paged)
    return cache, hc


def _fused_case(ora, D=128, bk=4, bv=2, G=64, gv=0, gq=4, n_new=1, lens=(200, 70, 129),
                dtype=torch.bfloat16, q_dtype=torch.bfloat16, split=None, rotate=False,
                page_size=0, cap=256, max_len=None):
    B, Hkv = len(lens), 2
    cache, hc = _make(ora, B, Hkv, D, cap, bk, bv, G, gv, rotate, page_size, list(lens))
    _prefill(ora, cache, hc, [max(0, n - n_new) for n in lens], D, seed=n_new + bk, dtype=dtype)
    k, v = _inputs(B, Hkv, n_new, D, seed=100 + n_new, dtype=dtype)
    q = torch.randn(B, Hkv * gq, D, generator=torch.Generator().manual_seed(gq)).to(q_dtype)
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    qb, qdt = workloads.as_bits(q)
    T = max_len or max(lens)
    ref, flags = ora.append_decode_attention(hc, kb, vb, qb, Hkv * gq, list(lens), dtype=dt,
                                             q_dtype=qdt, max_len=T)
    with _Split(split):
        out = kvq.kvq_append_decode_attention(
            cache, k.cuda(), v.cuda(), q.cuda(),
            torch.tensor(lens, dtype=torch.int32, device="cuda"), T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return cache, hc, out, ref, flags, (k, v, q, T)


@pytest.mark.parametrize("n_new", [1, 5, 16, 37])
@pytest.mark.parametrize("split", [None, 64, "balanced"])
@pytest.mark.parametrize("gq", [4, 16])
def test_fused_matches_oracle(ora, n_new, split, gq):
    # lengths put new tokens across the 64-position split boundaries
    cache, hc, out, ref, flags, _ = _fused_case(ora, gq=gq, n_new=n_new, split=split,
                                                lens=(130, 66, 256))
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_fused_input_types(ora, dtype):
    cache, hc, out, ref, flags, _ = _fused_case(ora, n_new=3, dtype=dtype, split=64)
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


@pytest.mark.parametrize("D,bk,bv,G,gv", [(64, 4, 2, 32, 0), (64, 8, 8, 64, 0),
                                          (128, 2, 4, 32, 128), (128, 8, 4, 128, 0),
                                          (128, 4, 2, 32, 64)])
def test_fused_other_shapes(ora, D, bk, bv, G, gv):
    cache, hc, out, ref, flags, _ = _fused_case(ora, D=D, bk=bk, bv=bv, G=G, gv=gv, n_new=9,
                                                split=64, q_dtype=torch.float32)
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


def test_fused_rotated_keys(ora):
    cache, hc, out, ref, flags, _ = _fused_case(ora, n_new=7, split=64, rotate=True)
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


@pytest.mark.parametrize("page_size", [32, 128])
def test_fused_paged(ora, page_size):
    cache, hc, out, ref, flags, _ = _fused_case(ora, n_new=16, split=64, page_size=page_size,
                                                lens=(200, 33, 256))
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


def test_rows_that_append_nothing(ora):
    # row 0 shorter than the append (flagged), row 1 longer than max_len
    # (clamped, flagged), row 2 normal
    cache, hc, out, ref, flags, _ = _fused_case(ora, n_new=8, lens=(3, 250, 100), max_len=200)
    assert flags == kvq.KVQ_DEVERR_BAD_POS | kvq.KVQ_DEVERR_SEQ_LEN
    assert kvq.kvq_device_error_flags() == flags
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


@pytest.mark.parametrize("split", [None, 64, "balanced"])
def test_fused_equals_two_calls(ora, split):
    # the fused call writes the same bytes as the append kernel and returns
    # the same bits as the separate decode
    B, Hkv, D, cap, n_new = 3, 2, 128, 512, 16
    lens = [500, 17, 300]
    fused = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    sep = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    kp, vp = _inputs(B, Hkv, cap, D, seed=1)
    for c in (fused, sep):
        kvq.kvq_quantize_append(c, kp.cuda(), vp.cuda(),
                                torch.zeros(B, dtype=torch.int32, device="cuda"))
    k, v = _inputs(B, Hkv, n_new, D, seed=2)
    q = torch.randn(B, 8 * Hkv, D, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    with _Split(split):
        a = kvq.kvq_append_decode_attention(fused, k.cuda(), v.cuda(), q.cuda(), lens_t, cap)
        kvq.kvq_quantize_append(sep, k.cuda(), v.cuda(),
                                torch.tensor([n - n_new for n in lens], dtype=torch.int32,
                                             device="cuda"))
        b = kvq.kvq_decode_attention(sep, q.cuda(), lens_t, cap)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error_flags() == 0
    for x, y in ((fused.k_codes, sep.k_codes), (fused.v_codes, sep.v_codes),
                 (fused.k_params, sep.k_params), (fused.v_params, sep.v_params)):
        assert torch.equal(x, y)
    assert torch.equal(a, b)


def test_zero_new_tokens_is_plain_decode(ora):
    B, Hkv, D, cap = 2, 2, 128, 128
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    kp, vp = _inputs(B, Hkv, cap, D, seed=4)
    kvq.kvq_quantize_append(cache, kp.cuda(), vp.cuda(),
                            torch.zeros(B, dtype=torch.int32, device="cuda"))
    before = [t.clone() for t in (cache.k_codes, cache.v_codes)]
    q = torch.randn(B, 4 * Hkv, D, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    lens = torch.tensor([100, 128], dtype=torch.int32, device="cuda")
    empty = torch.zeros(B, Hkv, 0, D, dtype=torch.bfloat16, device="cuda")
    a = kvq.kvq_append_decode_attention(cache, empty, empty, q.cuda(), lens, cap)
    b = kvq.kvq_decode_attention(cache, q.cuda(), lens, cap)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert all(torch.equal(x, y) for x, y in zip(before, (cache.k_codes, cache.v_codes)))


@pytest.mark.parametrize("n_new,lens", [(100, (100, 230, 164)), (64, (64, 128, 65))])
def test_fused_append_spans_several_splits(ora, n_new, lens):
    # more new tokens than a split holds (64): several CTAs of one slot each
    # write their own part; rows whose length equals n_new append at 0
    cache, hc, out, ref, flags, _ = _fused_case(ora, n_new=n_new, split=64, lens=lens, gq=16)
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


def test_fused_everything_at_once(ora):
    # rotated keys, coarser value groups, paged pool, f16 inputs, fp32 queries
    cache, hc, out, ref, flags, _ = _fused_case(ora, G=32, gv=128, n_new=21, split=64,
                                                rotate=True, page_size=64, lens=(150, 21, 256),
                                                dtype=torch.float16, q_dtype=torch.float32)
    assert flags == 0 and kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    compare_attention(out, ref, TOL)


def test_fused_bad_page_is_flagged_not_followed(ora):
    B, Hkv, D, cap, P, n_new = 2, 2, 128, 256, 64, 8
    table = np.array([[0, 1, -1, 6], [2, 3, 4, 5]], np.int32)   # row 0: entries 2, 3 bad
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64, page_size=P, num_pages=6,
                                 block_table=torch.from_numpy(table))
    hc = ora.PagedHostCache(B, Hkv, D, cap, 4, 2, 64, P, 6, table)
    _prefill(ora, cache, hc, [120, 120], D, seed=9, dtype=torch.bfloat16)
    k, v = _inputs(B, Hkv, n_new, D, seed=10)
    q = torch.randn(B, 2 * Hkv, D, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    lens = [133, 128]   # row 0's new positions 125..132 reach entry 2
    kb, dt = workloads.as_bits(k)
    vb, _ = workloads.as_bits(v)
    qb, qdt = workloads.as_bits(q)
    ref, flags = ora.append_decode_attention(hc, kb, vb, qb, 2 * Hkv, lens, dtype=dt,
                                             q_dtype=qdt, max_len=cap)
    assert flags == kvq.KVQ_DEVERR_BAD_PAGE
    out = kvq.kvq_append_decode_attention(cache, k.cuda(), v.cuda(), q.cuda(),
                                          torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                          cap, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error_flags() == kvq.KVQ_DEVERR_BAD_PAGE
    assert_same_cache(cache, hc)          # the valid pages hold the same bytes
    compare_attention(out[1:], ref[1:], TOL)   # row 0's output is unspecified
