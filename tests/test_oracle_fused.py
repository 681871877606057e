"""Pins of the oracle's fused append + decode (a composition of the two
pinned operations): it must equal an explicit append at seq_lens - n_new
followed by decode attention, append nothing for rows that are too short
(flagged) or out of range, and leave the other rows' bytes alone."""
import numpy as np

D, HKV = 64, 2


def _kv(rng, B, n):
    return ((rng.standard_normal((B, HKV, n, D)) * 2).astype(np.float32),
            rng.standard_normal((B, HKV, n, D)).astype(np.float32))


def test_fused_equals_append_then_decode(ora):
    rng = np.random.default_rng(0)
    B, cap, n_new = 3, 128, 5
    lens = [70, 5, 128]
    a = ora.HostCache(B, HKV, D, cap, 4, 2, 32)
    b = ora.HostCache(B, HKV, D, cap, 4, 2, 32)
    pre_k, pre_v = _kv(rng, B, cap)
    for hc in (a, b):
        hc.quantize_append(pre_k, pre_v, [0, 0, 0])
    k, v = _kv(rng, B, n_new)
    q = rng.standard_normal((B, 4 * HKV, D)).astype(np.float32)
    out, flags = ora.append_decode_attention(a, k, v, q, 4 * HKV, lens)
    assert flags == 0
    assert b.quantize_append(k, v, [n - n_new for n in lens]) == 0
    ref, _ = b.decode_attention(q, 4 * HKV, lens)
    np.testing.assert_array_equal(out, ref)
    for x, y in ((a.k_codes, b.k_codes), (a.v_codes, b.v_codes), (a.k_params, b.k_params),
                 (a.v_params, b.v_params)):
        np.testing.assert_array_equal(x, y)


def test_short_and_clamped_rows_append_nothing(ora):
    rng = np.random.default_rng(1)
    B, cap, n_new = 3, 64, 8
    hc = ora.HostCache(B, HKV, D, cap, 4, 8, 32)
    k, v = _kv(rng, B, n_new)
    q = rng.standard_normal((B, HKV, D)).astype(np.float32)
    # row 0 shorter than the append, row 1 past max_len, row 2 normal
    out, flags = ora.append_decode_attention(hc, k, v, q, HKV, [3, 60, 40], max_len=48)
    assert flags == ora.DEVERR_BAD_POS | 2  # BAD_POS and SEQ_LEN
    per = hc.k_codes.size // B
    assert not hc.k_codes[:2 * per].any()            # rows 0 and 1 untouched
    assert hc.k_codes[2 * per:].any()
    row2 = hc.dequant_row(1, 2, 1, 39)
    assert np.abs(row2 - v[2, 1, 7]).max() < 0.05      # last new value landed at 39
