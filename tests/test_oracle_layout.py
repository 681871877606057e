"""Pins of the oracle's packed-cache placement.

1. Bijection: every code of a K row / V tile gets its own bit field and the
   fields tile the row / tile exactly (no overlap, no hole).
2. Fragment semantics: reading the bytes the oracle writes the way the
   decode kernel does -- each lane takes its words, each word yields 16/b
   two-code registers, and the registers are placed into the 16x16 A operand
   of an m16n8k16 tensor-core instruction following the PTX fragment table
   (lane = 4*groupID + threadID_in_group; a0 = (row g, cols 2c..2c+1),
   a1 = (row g+8, ...), a2 = (row g, cols 2c+8..2c+9), a3 = (row g+8, ...))
   -- must rebuild the code matrix: tokens x dims for K (scores = K q),
   dims x tokens for V (output = V^T p).
3. Round trip through ora_quantize_append / ora_read_codes, and appends that
   leave neighbouring positions (including the other half of a shared V word)
   untouched.
"""
import numpy as np
import pytest

SHAPES = [(D, b) for D in (64, 128) for b in (2, 4, 8)]


@pytest.mark.parametrize("D,b", SHAPES)
def test_k_row_fields_tile_the_row(ora, D, b):
    used = np.zeros(D * b // 8 * 8, bool)
    for d in range(D):
        off, sh = ora.k_code_place(D, b, d)
        assert 0 <= off < D * b // 8 and sh + b <= 8
        bits = np.arange(off * 8 + sh, off * 8 + sh + b)
        assert not used[bits].any()
        used[bits] = True
    assert used.all()


@pytest.mark.parametrize("D,b", SHAPES)
def test_v_tile_fields_tile_the_tile(ora, D, b):
    nbytes = 2 * D * b
    used = np.zeros(nbytes * 8, bool)
    for k in range(16):
        for d in range(D):
            off, sh = ora.v_code_place(D, b, k, d)
            assert 0 <= off < nbytes and sh + b <= 8
            bits = np.arange(off * 8 + sh, off * 8 + sh + b)
            assert not used[bits].any()
            used[bits] = True
    assert used.all()


def _fragment_rows_cols(reg, g, c):
    """(row, col of the low half) of A-fragment register reg for lane (g, c)."""
    row = g + 8 * (reg & 1)
    col = 2 * c + 8 * (reg >> 1)
    return row, col


def _field(word, b, e, half):
    return (int(word) >> (16 * half + b * e)) & ((1 << b) - 1)


@pytest.mark.parametrize("D,b", SHAPES)
def test_k_rows_feed_score_fragments(ora, D, b):
    rng = np.random.default_rng(D * 10 + b)
    G = 32
    cache = ora.HostCache(1, 1, D, 16, b, 2, G)
    x = rng.standard_normal((1, 1, 16, D)).astype(np.float32)
    cache.quantize_append(x, x, [0])
    codes = np.stack([cache.read_codes(0, 0, 0, p) for p in range(16)])  # [token][dim]
    rows = cache.k_codes.reshape(16, D * b // 8)
    E = 16 // b
    slice_bytes = D * b // 32
    A = -np.ones((16, D), int)
    for lane in range(32):
        g, c = lane // 4, lane % 4
        for tok_half in (0, 1):               # token g (a0/a2) or g+8 (a1/a3)
            tok = g + 8 * tok_half
            words = rows[tok, c * slice_bytes:(c + 1) * slice_bytes].view(np.uint32)
            for i in range(D // 8):           # register i -> k-step i//2, cols +8*(i%2)
                w, e = divmod(i, E)
                kstep, s = divmod(i, 2)
                reg = tok_half + 2 * s
                row, col = _fragment_rows_cols(reg, g, c)
                assert row == tok
                for half in (0, 1):
                    A[row, 16 * kstep + col + half] = _field(words[w], b, e, half)
    assert np.array_equal(A, codes)


@pytest.mark.parametrize("D,b", SHAPES)
def test_v_tiles_feed_output_fragments(ora, D, b):
    rng = np.random.default_rng(D * 100 + b)
    cache = ora.HostCache(1, 1, D, 32, 2, b, 32)
    x = rng.standard_normal((1, 1, 32, D)).astype(np.float32)
    cache.quantize_append(x, x, [0])
    for tile in range(2):
        codes = np.stack([cache.read_codes(1, 0, 0, 16 * tile + k) for k in range(16)])
        tb = cache.v_codes[tile * 2 * D * b:(tile + 1) * 2 * D * b]
        N = D * b // 16
        P = min(16, N)
        E = 16 // b
        W = D * b // 128
        AT = -np.ones((D, 16), int)           # [dim][token in tile]
        for lane in range(32):
            g, c = lane // 4, lane % 4
            lane_bytes = np.array([tb[(n // P) * 32 * P + lane * P + n % P] for n in range(N)],
                                  np.uint8)
            words = lane_bytes.view(np.uint32)
            for u in (0, 1):                  # token columns 2c.. or 2c+8..
                for i in range(D // 8):       # register i -> m-tile i//2, rows +8*(i%2)
                    w, e = divmod(i, E)
                    mtile, v = divmod(i, 2)
                    reg = v + 2 * u
                    row, col = _fragment_rows_cols(reg, g, c)
                    for half in (0, 1):
                        AT[16 * mtile + row, col + half] = _field(words[u * W + w], b, e, half)
        assert np.array_equal(AT, codes.T)


@pytest.mark.parametrize("pos,n", [(0, 1), (5, 1), (15, 2), (16, 16), (3, 29), (31, 1)])
def test_append_preserves_other_positions(ora, pos, n):
    D, G = 128, 64
    rng = np.random.default_rng(pos * 7 + n)
    cache = ora.HostCache(2, 2, D, 48, 4, 2, G)
    base = rng.standard_normal((2, 2, 48, D)).astype(np.float32)
    assert cache.quantize_append(base, base * 0.5, [0, 0]) == 0
    before = {w: [[cache.read_codes(w, b, h, p) for p in range(48)] for b in range(2)
                  for h in range(2)] for w in (0, 1)}
    new = rng.standard_normal((2, 2, n, D)).astype(np.float32) * 3
    assert cache.quantize_append(new, new + 1, [pos, pos]) == 0
    for which in (0, 1):
        src = new if which == 0 else new + 1
        for b in range(2):
            for h in range(2):
                for p in range(48):
                    got = cache.read_codes(which, b, h, p)
                    if pos <= p < pos + n:
                        want = np.concatenate([
                            ora.quantize_group(src[b, h, p - pos, g * G:(g + 1) * G],
                                               4 if which == 0 else 2)[0] for g in range(2)])
                    else:
                        want = before[which][b * 2 + h][p]
                    assert np.array_equal(got, want), (which, b, h, p)


def test_append_past_capacity_is_skipped(ora):
    cache = ora.HostCache(2, 1, 64, 16, 4, 2, 32)
    x = np.ones((2, 1, 4, 64), np.float32)
    flags = cache.quantize_append(x, x, [14, 0])   # row 0 would pass 16
    assert flags == 1
    # row 0 untouched (params still zero), row 1 written
    ng = 2
    assert not cache.k_params[: 16 * ng * 2].any()
    assert cache.k_params[16 * ng * 2:].any()
    assert cache.quantize_append(x, x, [-1, 0]) == 8
