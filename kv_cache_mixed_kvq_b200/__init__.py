"""Key-priority mixed-precision KV-cache quantization and decode attention for B200.

Thin ctypes binding over ``libkvq.so`` (the C ABI in ``include/kvq.h``).  The
functions keep the C names; arguments are marshalled from torch tensors
(device pointers) and the current CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no fallback: if the library is
missing, every call raises.

Typical use::

    cache = KVCache.allocate(batch, kv_heads, head_dim, capacity,
                             bits_k=4, bits_v=2, group=64, device="cuda")
    kvq_quantize_append(cache, k, v, pos)            # k, v: [B][Hkv][n][D]
    out = kvq_decode_attention(cache, q, seq_lens, max_seq_len)   # q: [B][Hq][D]
    # or both in one launch, the new rows at seq_lens - n .. seq_lens - 1:
    out = kvq_append_decode_attention(cache, k, v, q, seq_lens, max_seq_len)

A paged cache (block tables) is allocated with ``page_size``, ``num_pages``
and an int32 ``block_table`` [batch][capacity / page_size].
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_F32, KVQ_BF16, KVQ_F16 = 0, 1, 2
KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = range(5)
KVQ_DEVERR_CAPACITY, KVQ_DEVERR_SEQ_LEN, KVQ_DEVERR_TIMEOUT, KVQ_DEVERR_BAD_POS = 1, 2, 4, 8
KVQ_DEVERR_BAD_PAGE = 16
KVQ_K_CODES, KVQ_V_CODES, KVQ_K_PARAMS, KVQ_V_PARAMS = range(4)
KVQ_FLAG_ROTATE_KEYS, KVQ_FLAG_PAGED = 1, 2

_DTYPE = {torch.float32: KVQ_F32, torch.bfloat16: KVQ_BF16, torch.float16: KVQ_F16}


class KvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {kvq_strerror(status)} (status {status})")
        self.status = status


class KvqCacheDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32),
        ("bits_k", ctypes.c_int32), ("bits_v", ctypes.c_int32),
        ("group", ctypes.c_int32), ("flags", ctypes.c_int32),
        ("group_v", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_params", ctypes.c_void_p), ("v_params", ctypes.c_void_p),
        ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
    ]


_lib = None


def library() -> ctypes.CDLL:
    """The loaded libkvq.so; raises if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY_PATH):
        raise RuntimeError(
            f"{LIBRARY_PATH} is missing: build it with `python -m kv_cache_mixed_kvq_b200.build`")
    lib = ctypes.CDLL(LIBRARY_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(KvqCacheDesc)
    lib.kvq_cache_bytes.argtypes = [I32] * 8
    lib.kvq_cache_bytes.restype = SZ
    lib.kvq_validate_cache.argtypes = [D]
    lib.kvq_validate_cache.restype = ctypes.c_int
    lib.kvq_quantize_append.argtypes = [D, P, P, I32, P, I32, P]
    lib.kvq_quantize_append.restype = ctypes.c_int
    lib.kvq_decode_workspace_bytes.argtypes = [D, I32, I32]
    lib.kvq_decode_workspace_bytes.restype = SZ
    lib.kvq_decode_split_tokens.argtypes = [D, I32, I32]
    lib.kvq_decode_split_tokens.restype = I32
    lib.kvq_decode_attention.argtypes = [D, P, I32, I32, P, I32, ctypes.c_float, P, I32, P, SZ, P]
    lib.kvq_decode_attention.restype = ctypes.c_int
    lib.kvq_append_decode_attention.argtypes = [D, P, P, I32, I32, P, I32, I32, P, I32,
                                                ctypes.c_float, P, I32, P, SZ, P]
    lib.kvq_append_decode_attention.restype = ctypes.c_int
    lib.kvq_device_error_flags.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.kvq_device_error_flags.restype = ctypes.c_int
    lib.kvq_last_device_error.argtypes = [P]
    lib.kvq_last_device_error.restype = ctypes.c_int
    lib.kvq_debug_inject_wait_timeout.argtypes = [I32, ctypes.c_int64]
    lib.kvq_debug_inject_wait_timeout.restype = ctypes.c_int
    lib.kvq_strerror.argtypes = [I32]
    lib.kvq_strerror.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check(status: int, what: str) -> None:
    if status != KVQ_OK:
        raise KvqError(status, what)


# ------------------------------------------------------------- C-named calls
def kvq_strerror(status: int) -> str:
    return library().kvq_strerror(int(status)).decode()


def kvq_cache_bytes(batch, kv_heads, head_dim, capacity, bits_k, bits_v, group, which) -> int:
    return int(library().kvq_cache_bytes(batch, kv_heads, head_dim, capacity, bits_k, bits_v,
                                         group, which))


@dataclasses.dataclass
class KVCache:
    """One layer's packed cache: four caller-owned device buffers + shape."""
    batch: int
    kv_heads: int
    head_dim: int
    capacity: int
    bits_k: int
    bits_v: int
    group: int
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_params: torch.Tensor
    v_params: torch.Tensor
    rotate_keys: bool = False  # KVQ_FLAG_ROTATE_KEYS: keys stored as H k
    group_v: int = 0           # values' group size (0: same as group)
    # KVQ_FLAG_PAGED: a pool of num_pages pages of page_size positions and an
    # int32 block table [batch][capacity / page_size] (device); 0 / None: slots
    page_size: int = 0
    num_pages: int = 0
    block_table: Optional[torch.Tensor] = None

    @classmethod
    def allocate(cls, batch, kv_heads, head_dim, capacity, bits_k, bits_v, group,
                 device="cuda", rotate_keys: bool = False, group_v: int = 0,
                 page_size: int = 0, num_pages: int = 0,
                 block_table: Optional[torch.Tensor] = None) -> "KVCache":
        """Zeroed buffers.  With page_size > 0 the cache is paged: a pool of
        num_pages pages and the given block table (int32 [batch][capacity /
        page_size], moved to `device`)."""
        gv = group_v or group
        rows, length = (num_pages, page_size) if page_size else (batch, capacity)
        sizes = [kvq_cache_bytes(rows, kv_heads, head_dim, length, bits_k, bits_v,
                                 gv if w == KVQ_V_PARAMS else group, w) for w in range(4)]
        if 0 in sizes:
            raise KvqError(KVQ_ERR_INVALID_ARG, "KVCache.allocate")
        if page_size:
            if block_table is None or capacity % page_size:
                raise KvqError(KVQ_ERR_INVALID_ARG, "KVCache.allocate (paged)")
            block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
            if tuple(block_table.shape) != (batch, capacity // page_size):
                raise KvqError(KVQ_ERR_INVALID_ARG, "KVCache.allocate (block table shape)")
        bufs = [torch.zeros(n, dtype=torch.uint8, device=device) for n in sizes]
        return cls(batch, kv_heads, head_dim, capacity, bits_k, bits_v, group, *bufs,
                   rotate_keys=rotate_keys, group_v=group_v, page_size=page_size,
                   num_pages=num_pages if page_size else 0,
                   block_table=block_table if page_size else None)

    def desc(self) -> KvqCacheDesc:
        flags = (KVQ_FLAG_ROTATE_KEYS if self.rotate_keys else 0) | \
            (KVQ_FLAG_PAGED if self.page_size else 0)
        bt = _dev_ptr(self.block_table, "block_table") if self.block_table is not None else None
        return KvqCacheDesc(self.batch, self.kv_heads, self.head_dim, self.capacity,
                            self.bits_k, self.bits_v, self.group, flags, self.group_v, 0,
                            _dev_ptr(self.k_codes, "k_codes"), _dev_ptr(self.v_codes, "v_codes"),
                            _dev_ptr(self.k_params, "k_params"), _dev_ptr(self.v_params, "v_params"),
                            self.page_size, self.num_pages, bt)


def kvq_validate_cache(cache: KVCache) -> int:
    d = cache.desc()
    return int(library().kvq_validate_cache(ctypes.byref(d)))


def kvq_quantize_append(cache: KVCache, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                        stream: Optional[torch.cuda.Stream] = None) -> None:
    """Quantize k, v ([B][Hkv][n_new][D]) into positions pos[b] .. pos[b]+n_new-1."""
    if k.dtype != v.dtype or k.shape != v.shape or k.dim() != 4:
        raise ValueError("k and v must be [B][Hkv][n_new][D] tensors of one dtype")
    if pos.dtype != torch.int32:
        raise ValueError("pos must be int32")
    d = cache.desc()
    st = library().kvq_quantize_append(ctypes.byref(d), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                       _DTYPE[k.dtype], _dev_ptr(pos, "pos"), k.shape[2],
                                       _stream_ptr(stream))
    _check(st, "kvq_quantize_append")


def kvq_decode_workspace_bytes(cache: KVCache, num_q_heads: int, max_seq_len: int) -> int:
    d = cache.desc()
    return int(library().kvq_decode_workspace_bytes(ctypes.byref(d), num_q_heads, max_seq_len))


def kvq_decode_split_tokens(cache: KVCache, num_q_heads: int, max_seq_len: int) -> int:
    d = cache.desc()
    return int(library().kvq_decode_split_tokens(ctypes.byref(d), num_q_heads, max_seq_len))


def kvq_decode_attention(cache: KVCache, q: torch.Tensor, seq_lens: torch.Tensor,
                         max_seq_len: int, sm_scale: float = 0.0,
                         out: Optional[torch.Tensor] = None,
                         out_dtype: Optional[torch.dtype] = None,
                         workspace: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Attention of q ([B][Hq][D]) over positions [0, seq_lens[b]) of the cache."""
    if q.dim() != 3:
        raise ValueError("q must be [B][Hq][D]")
    if seq_lens.dtype != torch.int32:
        raise ValueError("seq_lens must be int32")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    d = cache.desc()
    lib = library()
    if workspace is None:  # (a given workspace is checked by the library itself)
        need = int(lib.kvq_decode_workspace_bytes(ctypes.byref(d), q.shape[1], max_seq_len))
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev_ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.kvq_decode_attention(ctypes.byref(d), _dev_ptr(q, "q"), _DTYPE[q.dtype], q.shape[1],
                                  _dev_ptr(seq_lens, "seq_lens"), int(max_seq_len),
                                  float(sm_scale), _dev_ptr(out, "out"), _DTYPE[out.dtype],
                                  ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(st, "kvq_decode_attention")
    return out


def kvq_append_decode_attention(cache: KVCache, k_new: torch.Tensor, v_new: torch.Tensor,
                                q: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                                sm_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                out_dtype: Optional[torch.dtype] = None,
                                workspace: Optional[torch.Tensor] = None,
                                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Append k_new, v_new ([B][Hkv][n_new][D]) at positions seq_lens[b] - n_new ..
    seq_lens[b] - 1, then attend q ([B][Hq][D]) to [0, seq_lens[b]): one fused call."""
    if k_new.dtype != v_new.dtype or k_new.shape != v_new.shape or k_new.dim() != 4:
        raise ValueError("k_new and v_new must be [B][Hkv][n_new][D] tensors of one dtype")
    if q.dim() != 3:
        raise ValueError("q must be [B][Hq][D]")
    if seq_lens.dtype != torch.int32:
        raise ValueError("seq_lens must be int32")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    d = cache.desc()
    lib = library()
    if workspace is None:  # (a given workspace is checked by the library itself)
        need = int(lib.kvq_decode_workspace_bytes(ctypes.byref(d), q.shape[1], max_seq_len))
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev_ptr(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.kvq_append_decode_attention(
        ctypes.byref(d), _dev_ptr(k_new, "k_new"), _dev_ptr(v_new, "v_new"), _DTYPE[k_new.dtype],
        k_new.shape[2], _dev_ptr(q, "q"), _DTYPE[q.dtype], q.shape[1],
        _dev_ptr(seq_lens, "seq_lens"), int(max_seq_len), float(sm_scale), _dev_ptr(out, "out"),
        _DTYPE[out.dtype], ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(st, "kvq_append_decode_attention")
    return out


def kvq_debug_inject_wait_timeout(drop_stage: int, wait_limit_ns: int = 1_000_000) -> None:
    """Test knob: in the next decode launch, stage drop_stage (0 or 1) of the
    first warp's copy pipeline expects more bytes than its copies bring, so
    that a bounded wait runs out (see kvq.h); drop_stage < 0 disarms it."""
    _check(library().kvq_debug_inject_wait_timeout(int(drop_stage), int(wait_limit_ns)),
           "kvq_debug_inject_wait_timeout")


def kvq_device_error_flags(stream: Optional[torch.cuda.Stream] = None) -> int:
    flags = ctypes.c_uint32(0)
    st = library().kvq_device_error_flags(_stream_ptr(stream), ctypes.byref(flags))
    _check(st, "kvq_device_error_flags")
    return int(flags.value)


def kvq_last_device_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Error-word bits (read and cleared); raises KvqError on a CUDA failure."""
    r = library().kvq_last_device_error(_stream_ptr(stream))
    if r < 0:
        _check(-r, "kvq_last_device_error")
    return int(r)
