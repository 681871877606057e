"""Pins of the oracle's paged layout (block tables).

The summary page has no paged cache; the layout is the serving-system variant
of the cache format and is defined by its mapping alone: position p of batch
row b is local position p mod P of page block_table[b][p // P], and each
(page, kv head) is laid out like a slot of P positions.  These tests pin the
oracle's gather/scatter against that definition: byte by byte against an
independent slot-layout cache fed the same appends, with block tables that
permute pages, leave pool pages unused and share prefix pages.
"""
import numpy as np
import pytest

from kv_cache_mixed_kvq_b200 import workloads

D, HKV = 64, 2


def _kv(rng, B, n):
    k = (rng.standard_normal((B, HKV, n, D)) * 2).astype(np.float32)
    v = rng.standard_normal((B, HKV, n, D)).astype(np.float32)
    return k, v


def _pair(ora, B, cap, P, table, num_pages, bits=(4, 2), G=32, rotate=False):
    paged = ora.PagedHostCache(B, HKV, D, cap, bits[0], bits[1], G, P, num_pages, table,
                               rotate_keys=rotate)
    slots = ora.HostCache(B, HKV, D, cap, bits[0], bits[1], G, rotate_keys=rotate)
    return paged, slots


def _page_bytes(ora_cache, which, page):
    a = ora_cache.arrays[which]
    return a.reshape(ora_cache.num_pages, -1)[page]


def _slot_bytes(hc, which, b, h, j, P):
    a = (hc.k_codes, hc.v_codes, hc.k_params, hc.v_params)[which]
    per_slot = a.reshape(hc.B, hc.Hkv, -1)[b, h]
    L = per_slot.size // (hc.cap // P)
    return per_slot[j * L:(j + 1) * L]


@pytest.mark.parametrize("P", [32, 64])
def test_pages_hold_exactly_the_slot_bytes(ora, P):
    rng = np.random.default_rng(P)
    B, cap = 3, 128
    npg = cap // P
    num_pages = B * npg + 3                      # three pool pages stay unused
    table = rng.permutation(num_pages)[:B * npg].reshape(B, npg)
    paged, slots = _pair(ora, B, cap, P, table, num_pages)
    for pos, n in (([0, 5, 17], 40), ([40, 45, 57], 51)):
        k, v = _kv(rng, B, n)
        assert paged.quantize_append(k, v, pos) == slots.quantize_append(k, v, pos) == 0
    for which in range(4):
        for b in range(B):
            for j in range(npg):
                page_view = _page_bytes(paged, which, table[b][j]).reshape(HKV, -1)
                for h in range(HKV):
                    np.testing.assert_array_equal(page_view[h], _slot_bytes(slots, which, b, h, j, P))
        unused = sorted(set(range(num_pages)) - set(table.ravel()))
        for page in unused:
            assert not _page_bytes(paged, which, page).any()


def test_dequant_and_decode_follow_the_block_table(ora):
    rng = np.random.default_rng(5)
    B, cap, P = 2, 192, 32
    npg = cap // P
    num_pages = B * npg
    table = rng.permutation(num_pages).reshape(B, npg)
    paged, slots = _pair(ora, B, cap, P, table, num_pages, bits=(8, 4))
    k, v = _kv(rng, B, 150)
    paged.quantize_append(k, v, [0, 0])
    slots.quantize_append(k, v, [0, 0])
    for which in (0, 1):
        for b in range(B):
            for p in (0, 31, 32, 95, 149):
                np.testing.assert_array_equal(paged.dequant_row(which, b, 1, p),
                                              slots.dequant_row(which, b, 1, p))
    q = rng.standard_normal((B, 4 * HKV, D)).astype(np.float32)
    lens = [150, 77]
    a, fa = paged.decode_attention(q, 4 * HKV, lens)
    s, fs = slots.decode_attention(q, 4 * HKV, lens)
    assert fa == fs == 0
    np.testing.assert_array_equal(a, s)


def test_shared_prefix_pages(ora):
    # two rows share their first page (a common prefix) and own the rest
    rng = np.random.default_rng(9)
    cap, P = 128, 32
    table = np.array([[0, 1, 2, 3], [0, 4, 5, 6]])
    paged = ora.PagedHostCache(2, HKV, D, cap, 4, 2, 32, P, 7, table)
    # the prefix is written once, through row 0 alone (same pool)
    k0, v0 = _kv(rng, 1, 32)
    row0 = ora.PagedHostCache(1, HKV, D, cap, 4, 2, 32, P, 7, table[:1])
    row0.pool = paged.pool
    assert row0.quantize_append(k0, v0, [0]) == 0
    k1, v1 = _kv(rng, 2, 50)
    assert paged.quantize_append(k1, v1, [32, 32]) == 0
    # reference: a slot cache where both rows hold the prefix and their tokens
    ref = ora.HostCache(2, HKV, D, cap, 4, 2, 32)
    ref.quantize_append(np.concatenate([k0, k0]), np.concatenate([v0, v0]), [0, 0])
    ref.quantize_append(k1, v1, [32, 32])
    q = rng.standard_normal((2, 2 * HKV, D)).astype(np.float32)
    a, _ = paged.decode_attention(q, 2 * HKV, [82, 70])
    r, _ = ref.decode_attention(q, 2 * HKV, [82, 70])
    np.testing.assert_array_equal(a, r)


def test_bad_page_entries(ora):
    rng = np.random.default_rng(2)
    cap, P = 128, 32
    table = np.array([[0, 1, -1, 9], [2, 3, 4, 5]])   # row 0: pages 2 and 3 invalid
    paged = ora.PagedHostCache(2, HKV, D, cap, 4, 2, 32, P, 6, table)
    k, v = _kv(rng, 2, 60)
    # row 0 reaches only its pages 0 and 1: no flag
    assert paged.quantize_append(k, v, [0, 0]) == 0
    # row 0 reaches page 2 (entry -1): flagged, the valid pages still written
    k2, v2 = _kv(rng, 2, 20)
    flags = paged.quantize_append(k2, v2, [60, 60])
    assert flags == ora.DEVERR_BAD_PAGE
    q = rng.standard_normal((2, HKV, D)).astype(np.float32)
    assert paged.decode_attention(q, HKV, [64, 80])[1] == 0
    assert paged.decode_attention(q, HKV, [65, 80])[1] == ora.DEVERR_BAD_PAGE
    # a rejected append (past capacity) reaches no page
    assert paged.quantize_append(k2, v2, [120, 0]) == ora.DEVERR_CAPACITY


def test_paged_rotated_keys_match_slots(ora):
    rng = np.random.default_rng(4)
    B, cap, P = 2, 64, 32
    table = np.array([[3, 0], [1, 2]])
    paged, slots = _pair(ora, B, cap, P, table, 4, rotate=True)
    k, v = _kv(rng, B, 45)
    paged.quantize_append(k, v, [3, 0])
    slots.quantize_append(k, v, [3, 0])
    for which in range(4):
        for b in range(B):
            for j in range(2):
                page_view = _page_bytes(paged, which, table[b][j]).reshape(HKV, -1)
                for h in range(HKV):
                    np.testing.assert_array_equal(page_view[h], _slot_bytes(slots, which, b, h, j, P))


def test_workload_page_tables_are_permutations():
    # the seeded block tables used by the GPU tests and the benchmark
    for lens, P in (([100, 3000, 17], 64), ([4096] * 4, 256)):
        table, num_pages = workloads.make_block_table(lens, 4096, P, seed=1)
        used = table[table >= 0]
        assert used.size == len(set(used.tolist())) == sum((n + P - 1) // P for n in lens)
        assert num_pages >= used.size and used.max() < num_pages
        for b, n in enumerate(lens):
            assert (table[b, :(n + P - 1) // P] >= 0).all()


# ------------------------------------------------- planted mistakes (mutants)
def _mutants(ora):
    Base = ora.PagedHostCache

    class IgnoresTable(Base):      # pages taken in row order, block table ignored
        def __init__(self, B, Hkv, D_, cap, bk, bv, g, P, num_pages, table, **kw):
            npg = cap // P
            ident = np.arange(B * npg).reshape(B, npg) % num_pages
            super().__init__(B, Hkv, D_, cap, bk, bv, g, P, num_pages, ident, **kw)

    class ShiftedPage(Base):       # logical page j mapped through entry j - 1
        def __init__(self, B, Hkv, D_, cap, bk, bv, g, P, num_pages, table, **kw):
            shifted = np.roll(np.array(table).reshape(B, cap // P), 1, axis=1)
            super().__init__(B, Hkv, D_, cap, bk, bv, g, P, num_pages, shifted, **kw)

    class NoWriteBack(Base):       # appends never reach the pool
        def _scatter(self, hc, b, pages):
            return None

    class NoBadPageFlag(Base):
        def quantize_append(self, *a, **kw):
            return super().quantize_append(*a, **kw) & ~ora.DEVERR_BAD_PAGE

    return {"ignores_table": IgnoresTable, "shifted_page": ShiftedPage,
            "no_write_back": NoWriteBack, "no_bad_page_flag": NoBadPageFlag}


PAGED_PINS = [
    lambda o: test_pages_hold_exactly_the_slot_bytes(o, 32),
    lambda o: test_dequant_and_decode_follow_the_block_table(o),
    lambda o: test_shared_prefix_pages(o),
    lambda o: test_bad_page_entries(o),
]


@pytest.mark.parametrize("name", ["ignores_table", "shifted_page", "no_write_back",
                                  "no_bad_page_flag"])
def test_some_pin_catches_the_paged_mutant(ora, monkeypatch, name):
    monkeypatch.setattr(ora, "PagedHostCache", _mutants(ora)[name])
    caught = 0
    for pin in PAGED_PINS:
        try:
            pin(ora)
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the mutant {name}"
