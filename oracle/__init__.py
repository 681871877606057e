"""CPU oracle for key-priority mixed-precision KV-cache quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (``kv_cache_mixed_kvq_b200``) never imports it and shares no code
with it: the C source next to this file restates the quantizer, the cache
format and attention from their definitions.

Functions follow "Quantize What Counts: More for Keys, Less for Values"
(summary page): keys and values quantized with separate bit widths
("Key contributions", K4V2 etc.), group-wise ("Results", "Group-size
sensitivity"), and attention over the dequantised cache ("Problem
statement": the cache is what inference reads).  See ``kvq_oracle.c`` for the
step-by-step definitions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

DTYPE_CODE = {"f32": 0, "bf16": 1, "f16": 2}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", _SRC, "-o", tmp, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _load(path: str | None = None):
    lib = ctypes.CDLL(path or build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.ora_f32_to_f16.argtypes = [ctypes.c_float]
    lib.ora_f32_to_f16.restype = ctypes.c_uint16
    lib.ora_f16_to_f32.argtypes = [ctypes.c_uint16]
    lib.ora_f16_to_f32.restype = ctypes.c_float
    lib.ora_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.ora_bf16_to_f32.restype = ctypes.c_float
    lib.ora_quantize_group.argtypes = [P, I, I, P, P, P, P, P]
    lib.ora_quantize_group.restype = None
    lib.ora_k_code_place.argtypes = [I, I, I, P, P]
    lib.ora_v_code_place.argtypes = [I, I, I, I, P, P]
    lib.ora_quantize_append.argtypes = [I] * 7 + [P] * 6 + [I, P, I]
    lib.ora_quantize_append.restype = I
    lib.ora_read_codes.argtypes = [I, I, I, I, I, P, P, I, I, I, I, P]
    lib.ora_dequant_row.argtypes = [I, I, I, I, I, I, P, P, P, P, I, I, I, I, P]
    lib.ora_decode_attention.argtypes = [I] * 7 + [P] * 4 + [P, I, I, P, I, ctypes.c_float, P]
    lib.ora_decode_attention.restype = I
    lib.ora_attention_dense.argtypes = [I, I, I, I, P, P, I, P, I, I, P, ctypes.c_float, P]
    lib.ora_attention_dense.restype = I
    lib.ora_fwht.argtypes = [P, I]
    lib.ora_fwht.restype = None
    lib.ora_quantize_append_ex.argtypes = [I] * 7 + [P] * 6 + [I, P, I, I]
    lib.ora_quantize_append_ex.restype = I
    lib.ora_decode_attention_ex.argtypes = [I] * 7 + [P] * 4 + [P, I, I, P, I, ctypes.c_float,
                                                              I, P]
    lib.ora_decode_attention_ex.restype = I
    lib.ora_quantize_append_g2.argtypes = [I] * 8 + [P] * 6 + [I, P, I, I]
    lib.ora_quantize_append_g2.restype = I
    lib.ora_decode_attention_g2.argtypes = [I] * 8 + [P] * 4 + [P, I, I, P, I, ctypes.c_float,
                                                              I, P]
    lib.ora_decode_attention_g2.restype = I
    return lib


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_of(a: np.ndarray, dtype: str | None) -> str:
    if dtype is not None:
        return dtype
    if a.dtype == np.float32:
        return "f32"
    raise ValueError("16-bit inputs are passed as uint16 bit patterns with dtype='bf16' or 'f16'")


# ------------------------------------------------------------------ numbers
def f32_to_f16_bits(x: float) -> int:
    return int(lib().ora_f32_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().ora_f16_to_f32(int(h)))


def bf16_bits_to_f32(h: int) -> float:
    return float(lib().ora_bf16_to_f32(int(h)))


# ---------------------------------------------------------------- quantizer
def quantize_group(x, bits: int):
    """Codes, binary32 scale and min, binary16 scale/zero bits of one group."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, np.uint8)
    s32 = np.zeros(1, np.float32)
    m32 = np.zeros(1, np.float32)
    s16 = np.zeros(1, np.uint16)
    z16 = np.zeros(1, np.uint16)
    lib().ora_quantize_group(_ptr(x), x.size, bits, _ptr(codes), _ptr(s32), _ptr(m32),
                             _ptr(s16), _ptr(z16))
    return codes, float(s32[0]), float(m32[0]), int(s16[0]), int(z16[0])


def k_code_place(D: int, bits: int, d: int):
    off = ctypes.c_int()
    sh = ctypes.c_int()
    lib().ora_k_code_place(D, bits, d, ctypes.byref(off), ctypes.byref(sh))
    return off.value, sh.value


def v_code_place(D: int, bits: int, k: int, d: int):
    off = ctypes.c_int()
    sh = ctypes.c_int()
    lib().ora_v_code_place(D, bits, k, d, ctypes.byref(off), ctypes.byref(sh))
    return off.value, sh.value


# ------------------------------------------------------------------- cache
class HostCache:
    """Host copies of the four cache arrays in the library's format."""

    def __init__(self, B, Hkv, D, capacity, bits_k, bits_v, group, rotate_keys=False,
                 group_v=None):
        self.B, self.Hkv, self.D, self.cap = B, Hkv, D, capacity
        self.bits_k, self.bits_v, self.group = bits_k, bits_v, group
        self.group_v = group if not group_v else group_v  # values' group size
        self.rotate_keys = bool(rotate_keys)  # keys stored as H k (Walsh-Hadamard)
        slots = B * Hkv
        self.k_codes = np.zeros(slots * capacity * D * bits_k // 8, np.uint8)
        self.v_codes = np.zeros(slots * capacity * D * bits_v // 8, np.uint8)
        ng = D // group
        self.k_params = np.zeros(slots * capacity * ng * 2, np.uint16)
        self.v_params = np.zeros(slots * capacity * (D // self.group_v) * 2, np.uint16)

    def _shape(self):
        return (self.B, self.Hkv, self.D, self.cap, self.bits_k, self.bits_v, self.group)

    def quantize_append(self, k: np.ndarray, v: np.ndarray, pos, dtype: str | None = None) -> int:
        """k, v: [B][Hkv][n_new][D] float32 or uint16 bit patterns."""
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        n_new = k.shape[2]
        assert k.shape == (self.B, self.Hkv, n_new, self.D) and v.shape == k.shape
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        dt = DTYPE_CODE[_dtype_of(k, dtype)]
        r = lib().ora_quantize_append_g2(*self._shape(), self.group_v, _ptr(self.k_codes),
                                         _ptr(self.v_codes), _ptr(self.k_params),
                                         _ptr(self.v_params), _ptr(k), _ptr(v), dt, _ptr(pos),
                                         n_new, int(self.rotate_keys))
        if r < 0:
            raise ValueError("invalid cache shape")
        return r

    def read_codes(self, which: int, b: int, h: int, p: int) -> np.ndarray:
        out = np.zeros(self.D, np.uint8)
        lib().ora_read_codes(self.Hkv, self.D, self.cap, self.bits_k, self.bits_v,
                             _ptr(self.k_codes), _ptr(self.v_codes), which, b, h, p, _ptr(out))
        return out

    def dequant_row(self, which: int, b: int, h: int, p: int) -> np.ndarray:
        out = np.zeros(self.D, np.float32)
        lib().ora_dequant_row(self.Hkv, self.D, self.cap, self.bits_k, self.bits_v,
                              self.group if which == 0 else self.group_v,
                              _ptr(self.k_codes), _ptr(self.v_codes), _ptr(self.k_params),
                              _ptr(self.v_params), which, b, h, p, _ptr(out))
        return out

    def dequant_slot(self, which: int, b: int, h: int, n: int) -> np.ndarray:
        return np.stack([self.dequant_row(which, b, h, p) for p in range(n)]) if n else \
            np.zeros((0, self.D), np.float32)

    def decode_attention(self, q: np.ndarray, Hq: int, seq_lens, sm_scale: float = 0.0,
                         q_dtype: str | None = None, max_len: int | None = None):
        """Returns (out float64 [B][Hq][D], flags)."""
        q = np.ascontiguousarray(q)
        assert q.shape == (self.B, Hq, self.D)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        out = np.zeros((self.B, Hq, self.D), np.float64)
        r = lib().ora_decode_attention_g2(*self._shape(), self.group_v, _ptr(self.k_codes),
                                          _ptr(self.v_codes),
                                       _ptr(self.k_params), _ptr(self.v_params), _ptr(q),
                                       DTYPE_CODE[_dtype_of(q, q_dtype)], Hq, _ptr(lens),
                                       self.cap if max_len is None else max_len,
                                       float(sm_scale), int(self.rotate_keys), _ptr(out))
        if r < 0:
            raise ValueError("invalid shape")
        return out, r


DEVERR_CAPACITY, DEVERR_BAD_POS, DEVERR_BAD_PAGE = 1, 8, 16


class PagedHostCache:
    """Paged variant (block tables) of HostCache.

    The summary page has no paged layout: this is the serving-system variant
    of the cache format, defined by its mapping alone.  A pool of
    ``num_pages`` pages of ``page_size`` (P) positions holds all kv heads of
    each page, and (page, kv head) is laid out exactly like a slot of P
    positions, so the pool is a HostCache of ``num_pages`` batch rows and
    capacity P.  Position p of batch row b is local position p mod P of page
    ``block_table[b][p // P]``.

    Every operation gathers each batch row's pages into a slot-layout
    HostCache of ``capacity`` positions, runs the slot operation there and
    scatters the pages back (batch rows one after another).  Block-table
    entries outside [0, num_pages) read as zero pages and are never written;
    reaching one sets DEVERR_BAD_PAGE.
    """

    def __init__(self, B, Hkv, D, capacity, bits_k, bits_v, group, page_size, num_pages,
                 block_table, rotate_keys=False, group_v=None):
        assert capacity % page_size == 0 and page_size % 16 == 0
        self.B, self.Hkv, self.D, self.cap, self.P = B, Hkv, D, capacity, page_size
        self.num_pages = num_pages
        self.shape = (D, bits_k, bits_v, group, rotate_keys, group_v)
        self.block_table = np.array(block_table, dtype=np.int64).reshape(B, capacity // page_size)
        self.pool = HostCache(num_pages, Hkv, D, page_size, bits_k, bits_v, group,
                              rotate_keys=rotate_keys, group_v=group_v)

    # the four arrays, page-major [num_pages][Hkv][...]
    @property
    def arrays(self):
        p = self.pool
        return [p.k_codes, p.v_codes, p.k_params, p.v_params]

    k_codes = property(lambda self: self.pool.k_codes)
    v_codes = property(lambda self: self.pool.v_codes)
    k_params = property(lambda self: self.pool.k_params)
    v_params = property(lambda self: self.pool.v_params)

    def _row_cache(self, rows: int) -> HostCache:
        D, bk, bv, g, rot, gv = self.shape
        return HostCache(rows, self.Hkv, D, self.cap, bk, bv, g, rotate_keys=rot, group_v=gv)

    def _views(self, hc: HostCache, rows: int):
        """(pool view [num_pages][Hkv][L], row view [rows][Hkv][pages per row][L])
        of each array, L the elements of P positions of one slot."""
        npg = self.cap // self.P
        out = []
        for pool_a, row_a in zip(self.arrays, (hc.k_codes, hc.v_codes, hc.k_params, hc.v_params)):
            L = pool_a.size // (self.num_pages * self.Hkv)
            out.append((pool_a.reshape(self.num_pages, self.Hkv, L),
                        row_a.reshape(rows, self.Hkv, npg, L)))
        return out

    def _valid(self, page) -> bool:
        return 0 <= page < self.num_pages

    def gather(self, rows=None) -> HostCache:
        """Slot-layout copy of the given batch rows (all by default)."""
        rows = list(range(self.B)) if rows is None else list(rows)
        hc = self._row_cache(len(rows))
        for pool_v, row_v in self._views(hc, len(rows)):
            for i, b in enumerate(rows):
                for j, page in enumerate(self.block_table[b]):
                    if self._valid(page):
                        row_v[i, :, j, :] = pool_v[page]
        return hc

    def _scatter(self, hc: HostCache, b: int, pages) -> None:
        for pool_v, row_v in self._views(hc, 1):
            for j in pages:
                page = self.block_table[b][j]
                if self._valid(page):
                    pool_v[page] = row_v[0, :, j, :]

    def quantize_append(self, k: np.ndarray, v: np.ndarray, pos, dtype: str | None = None) -> int:
        """As HostCache.quantize_append, through the block table."""
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        n_new = k.shape[2]
        flags = 0
        for b in range(self.B):
            hc = self.gather([b])
            r = hc.quantize_append(k[b:b + 1], v[b:b + 1], [int(pos[b])], dtype=dtype)
            flags |= r
            if r & (DEVERR_CAPACITY | DEVERR_BAD_POS) or n_new == 0:
                continue  # row rejected: nothing written, no page reached
            first = (int(pos[b]) // 16) * 16
            last = (int(pos[b]) + n_new + 15) // 16 * 16 - 1  # last position of the last tile
            pages = range(first // self.P, last // self.P + 1)
            if any(not self._valid(self.block_table[b][j]) for j in pages):
                flags |= DEVERR_BAD_PAGE
            self._scatter(hc, b, pages)
        return flags

    def decode_attention(self, q: np.ndarray, Hq: int, seq_lens, sm_scale: float = 0.0,
                         q_dtype: str | None = None, max_len: int | None = None):
        """As HostCache.decode_attention over the gathered rows; rows that
        reach an invalid page set DEVERR_BAD_PAGE (their output is not
        defined by the library)."""
        out, flags = self.gather().decode_attention(q, Hq, seq_lens, sm_scale=sm_scale,
                                                    q_dtype=q_dtype, max_len=max_len)
        lim = min(self.cap, self.cap if max_len is None else max_len)
        for b, n in enumerate(seq_lens):
            n = max(0, min(int(n), lim))
            if any(not self._valid(self.block_table[b][j]) for j in range((n + self.P - 1) // self.P)):
                flags |= DEVERR_BAD_PAGE
        return out, flags

    def dequant_row(self, which: int, b: int, h: int, p: int) -> np.ndarray:
        page = int(self.block_table[b][p // self.P])
        return self.pool.dequant_row(which, page, h, p % self.P)


def append_decode_attention(hc, k: np.ndarray, v: np.ndarray, q: np.ndarray, Hq: int, seq_lens,
                            dtype: str | None = None, q_dtype: str | None = None,
                            max_len: int | None = None, sm_scale: float = 0.0):
    """Definition of the fused append + decode call, as the composition of
    the two operations: every batch row b whose length n = seq_lens[b] is
    within min(capacity, max_len) appends its n_new new rows at positions
    n - n_new .. n - 1 (a row with n < n_new appends nothing and sets
    DEVERR_BAD_POS; a row with n out of range appends nothing and the
    decode flags it), then attention over [0, n).  `hc`: HostCache or
    PagedHostCache.  Returns (out, flags)."""
    n_new = k.shape[2]
    lim = min(hc.cap, hc.cap if max_len is None else max_len)
    lens = [int(n) for n in seq_lens]
    flags = 0
    # rows that append nothing get position `capacity` (past the end: the
    # append skips them); its capacity flag is not part of this call's result
    pos = []
    for n in lens:
        if n > lim:
            pos.append(hc.cap)
        elif n < n_new:
            flags |= DEVERR_BAD_POS
            pos.append(hc.cap)
        else:
            pos.append(n - n_new)
    skipped = any(p == hc.cap for p in pos)
    f = hc.quantize_append(k, v, pos, dtype=dtype)
    flags |= (f & ~DEVERR_CAPACITY) if skipped else f
    out, f2 = hc.decode_attention(q, Hq, lens, sm_scale=sm_scale, q_dtype=q_dtype,
                                  max_len=max_len)
    return out, flags | f2


def fwht(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform of a binary32 vector (the oracle's
    key rotation, same butterfly order and rounding)."""
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    lib().ora_fwht(_ptr(y), y.size)
    return y


def attention_dense(k: np.ndarray, v: np.ndarray, q: np.ndarray, seq_lens, sm_scale: float = 0.0,
                    kv_dtype: str | None = None, q_dtype: str | None = None) -> np.ndarray:
    """Unquantised attention: k, v [B][Hkv][T][D], q [B][Hq][D] -> float64."""
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    q = np.ascontiguousarray(q)
    B, Hkv, T, D = k.shape
    Hq = q.shape[1]
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    r = lib().ora_attention_dense(B, Hkv, D, T, _ptr(k), _ptr(v), DTYPE_CODE[_dtype_of(k, kv_dtype)],
                                  _ptr(q), DTYPE_CODE[_dtype_of(q, q_dtype)], Hq, _ptr(lens),
                                  float(sm_scale), _ptr(out))
    if r < 0:
        raise ValueError("invalid shape")
    return out
