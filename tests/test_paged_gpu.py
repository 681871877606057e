"""GPU parity of the paged cache layout (block tables, KVQ_FLAG_PAGED)
against the oracle's paged cache: the page pool must be bit-identical after
appends of any alignment (permuted pages, unused pool pages, page sizes 32 to
256, every bit pair, head_dim 64 and 128, rotated keys, separate value
groups), decode attention must match the binary64 oracle within 2e-3 with
splits that cross pages and with rows sharing prefix pages, and block-table
entries outside the pool must be flagged, never followed."""
import os

import numpy as np
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


def _paged_pair(ora, B, Hkv, D, cap, bk, bv, G, P, table, num_pages, gv=0, rotate=False):
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, bk, bv, G, group_v=gv, rotate_keys=rotate,
                                 page_size=P, num_pages=num_pages,
                                 block_table=torch.from_numpy(np.ascontiguousarray(table)))
    hc = ora.PagedHostCache(B, Hkv, D, cap, bk, bv, G, P, num_pages, table,
                            rotate_keys=rotate, group_v=gv or None)
    return cache, hc


def _decode(cache, q, lens, T, out_dtype=torch.float32):
    out = kvq.kvq_decode_attention(cache, q.cuda(), torch.tensor(lens, dtype=torch.int32,
                                                                 device="cuda"),
                                   T, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out


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


@pytest.mark.parametrize("P", [32, 64, 256])
@pytest.mark.parametrize("D,bk,bv,G", [(128, 4, 2, 64), (128, 8, 4, 32), (128, 2, 4, 64),
                                       (64, 4, 2, 32), (64, 8, 8, 64)])
def test_paged_cache_bit_exact(ora, P, D, bk, bv, G):
    B, Hkv, cap = 3, 2, 512
    lens = [300, 77, 512]
    table, num_pages = workloads.make_block_table(lens, cap, P, seed=P + D, spare=2)
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, bk, bv, G, P, table, num_pages)
    # every row's pages are written by two appends, the second mid-tile
    k, v = _inputs(B, Hkv, 70, D, seed=bk * 10 + bv)
    assert append(ora, cache, hc, k, v, [0, 0, 0]) == (0, 0)
    k, v = _inputs(B, Hkv, 7, D, seed=3)
    assert append(ora, cache, hc, k, v, [70, 70, 70]) == (0, 0)
    assert_same_cache(cache, hc)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_paged_input_types(ora, dtype):
    B, Hkv, D, cap, P = 2, 2, 128, 256, 64
    table, num_pages = workloads.make_block_table([256, 256], cap, P, seed=11)
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, 4, 2, 64, P, table, num_pages)
    for (pos, n), seed in zip([((0, 19), 100), ((100, 119), 60)], range(2)):
        k, v = _inputs(B, Hkv, n, D, seed=seed, dtype=dtype)
        assert append(ora, cache, hc, k, v, list(pos)) == (0, 0)
    assert_same_cache(cache, hc)


def test_paged_rotated_keys_and_value_groups(ora):
    B, Hkv, D, cap, P = 2, 2, 128, 320, 32
    table, num_pages = workloads.make_block_table([320, 200], cap, P, seed=4, spare=5)
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, 4, 2, 32, P, table, num_pages, gv=128,
                            rotate=True)
    k, v = _inputs(B, Hkv, 200, D, seed=8)
    assert append(ora, cache, hc, k, v, [0, 0]) == (0, 0)
    assert_same_cache(cache, hc)
    q = torch.randn(B, 4 * Hkv, D, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    ref, flags = hc.decode_attention(qb, 4 * Hkv, [200, 133], q_dtype=qdt, max_len=cap)
    assert flags == 0
    compare_attention(_decode(cache, q, [200, 133], cap), ref, TOL)


@pytest.mark.parametrize("split", [None, 64, 128, 448, "balanced"])
@pytest.mark.parametrize("P", [32, 128])
@pytest.mark.parametrize("gq,q_dtype", [(4, torch.bfloat16), (8, torch.float32)])
def test_paged_decode_matches_oracle(ora, split, P, gq, q_dtype):
    B, Hkv, D = 3, 2, 128
    lens = [700, 1, 333]
    cap = 768
    table, num_pages = workloads.make_block_table(lens, cap, P, seed=P + gq, spare=3)
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, 4, 2, 64, P, table, num_pages)
    k, v = _inputs(B, Hkv, max(lens), D, seed=gq)
    # rows append only up to their own length (their later pages are -1)
    for b in range(B):
        sub = ora.PagedHostCache(1, Hkv, D, cap, 4, 2, 64, P, num_pages, table[b:b + 1])
        sub.pool = hc.pool
        n = lens[b]
        kb, dt = workloads.as_bits(k[b:b + 1, :, :n])
        vb, _ = workloads.as_bits(v[b:b + 1, :, :n])
        assert sub.quantize_append(kb, vb, [0], dtype=dt) == 0
        one = kvq.KVCache(1, Hkv, D, cap, 4, 2, 64, cache.k_codes, cache.v_codes, cache.k_params,
                          cache.v_params, page_size=P, num_pages=num_pages,
                          block_table=cache.block_table[b:b + 1].contiguous())
        kvq.kvq_quantize_append(one, k[b:b + 1, :, :n].cuda(), v[b:b + 1, :, :n].cuda(),
                                torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert kvq.kvq_device_error_flags() == 0
    assert_same_cache(cache, hc)
    q = torch.randn(B, Hkv * gq, D, generator=torch.Generator().manual_seed(gq)).to(q_dtype)
    qb, qdt = workloads.as_bits(q)
    ref, flags = hc.decode_attention(qb, Hkv * gq, lens, q_dtype=qdt, max_len=max(lens))
    assert flags == 0
    with _Split(split):
        out = _decode(cache, q, lens, max(lens))
    assert kvq.kvq_device_error_flags() == 0
    compare_attention(out, ref, TOL)


def test_paged_decode_equals_slot_decode(ora):
    # the same rows in a slot cache and in a shuffled page pool: identical bits
    B, Hkv, D, cap, P = 2, 4, 128, 1024, 64
    lens = [1000, 513]
    table, num_pages = workloads.make_block_table([cap, cap], cap, P, seed=2)
    paged = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64, page_size=P, num_pages=num_pages,
                                 block_table=torch.from_numpy(table))
    slots = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    k, v = _inputs(B, Hkv, cap, D, seed=5)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    for c in (paged, slots):
        kvq.kvq_quantize_append(c, k.cuda(), v.cuda(), pos)
    q = torch.randn(B, 4 * Hkv, D, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    for split in (None, 64):
        with _Split(split):
            a = _decode(paged, q, lens, cap)
            b = _decode(slots, q, lens, cap)
        assert torch.equal(a, b)


def test_shared_prefix_pages_decode(ora):
    B, Hkv, D, cap, P = 2, 2, 128, 256, 64
    table = np.array([[0, 1, 2, 3], [0, 1, 4, 5]], np.int32)   # 128-token shared prefix
    num_pages = 6
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, 4, 2, 64, P, table, num_pages)
    # the prefix through row 0 alone, then both rows' own tokens
    one = kvq.KVCache(1, Hkv, D, cap, 4, 2, 64, cache.k_codes, cache.v_codes, cache.k_params,
                      cache.v_params, page_size=P, num_pages=num_pages,
                      block_table=cache.block_table[:1].contiguous())
    sub = ora.PagedHostCache(1, Hkv, D, cap, 4, 2, 64, P, num_pages, table[:1])
    sub.pool = hc.pool
    k0, v0 = _inputs(1, Hkv, 128, D, seed=1)
    assert append(ora, one, sub, k0, v0, [0]) == (0, 0)
    k1, v1 = _inputs(B, Hkv, 100, D, seed=2)
    assert append(ora, cache, hc, k1, v1, [128, 128]) == (0, 0)
    assert_same_cache(cache, hc)
    q = torch.randn(B, 4 * Hkv, D, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    ref, flags = hc.decode_attention(qb, 4 * Hkv, [228, 150], q_dtype=qdt, max_len=cap)
    assert flags == 0
    compare_attention(_decode(cache, q, [228, 150], cap), ref, TOL)


def test_bad_page_entries_are_flagged_not_followed(ora):
    B, Hkv, D, cap, P = 2, 2, 128, 256, 64
    table = np.array([[0, 1, -1, 7], [2, 3, 4, 5]], np.int32)   # row 0: entries 2, 3 bad
    num_pages = 6
    cache, hc = _paged_pair(ora, B, Hkv, D, cap, 4, 2, 64, P, table, num_pages)
    k, v = _inputs(B, Hkv, 100, D, seed=3)
    # row 0 reaches entry 2 (-1): its tiles there are skipped, the rest written
    fo, fg = append(ora, cache, hc, k, v, [60, 60])
    assert fo == fg == kvq.KVQ_DEVERR_BAD_PAGE
    assert_same_cache(cache, hc)
    q = torch.randn(B, 2 * Hkv, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    qb, qdt = workloads.as_bits(q)
    # decode of row 0 past its valid pages: flagged; row 1 unaffected
    ref, flags = hc.decode_attention(qb, 2 * Hkv, [150, 160], q_dtype=qdt, max_len=cap)
    assert flags == kvq.KVQ_DEVERR_BAD_PAGE
    out = _decode(cache, q, [150, 160], cap)
    assert kvq.kvq_device_error_flags() == kvq.KVQ_DEVERR_BAD_PAGE
    compare_attention(out[1:], ref[1:], TOL)
    # within the valid pages: no flag, and row 0 matches too
    ref, flags = hc.decode_attention(qb, 2 * Hkv, [128, 160], q_dtype=qdt, max_len=cap)
    assert flags == 0
    out = _decode(cache, q, [128, 160], cap)
    assert kvq.kvq_device_error_flags() == 0
    compare_attention(out, ref, TOL)
