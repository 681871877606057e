"""kvq_decode_attention_static(): decode attention without any allocation.

For callers that may not allocate device memory (engines that plan all
device memory up front, plain-C hosts without an allocator), the library
offers a variant whose split-K scratch is a fixed array in its device image.
This file is collected last on purpose.  It calls the variant through the C
ABI on a large multi-split shape and then twice in a row on a smaller one
(stale partials of another plan are left in the scratch), and checks that
each output equals the regular entry point's bit for bit: both run the same
split plan and the same deterministic kernels.  It also checks that a shape
needing more than the fixed scratch is refused.
"""
import ctypes

import pytest
import torch

import kv_cache_mixed_kvq_b200 as kvq

pytestmark = pytest.mark.gpu

STATIC_BYTES = 4 << 20


def _static_fn():
    fn = kvq.library().kvq_decode_attention_static
    fn.argtypes = [ctypes.POINTER(kvq.KvqCacheDesc), ctypes.c_void_p, ctypes.c_int32,
                   ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _filled_cache(B, Hkv, D, T, seed):
    g = torch.Generator().manual_seed(seed)
    cap = (T + 15) // 16 * 16
    cache = kvq.KVCache.allocate(B, Hkv, D, cap, 4, 2, 64)
    k = (torch.randn(B, Hkv, T, D, generator=g) * 2).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16).cuda()
    kvq.kvq_quantize_append(cache, k, v, torch.zeros(B, dtype=torch.int32, device="cuda"))
    return cache


def _static_vs_regular(fn, cache, Hq, lens, T, seed):
    """One call of each entry point on the same inputs; the static one must
    reproduce the regular one bit for bit (same plan, same kernels)."""
    B, D = cache.batch, cache.head_dim
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(seed)).to(
        torch.bfloat16).cuda()
    ref = kvq.kvq_decode_attention(cache, q, lens, T, out_dtype=torch.float32)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    desc = cache.desc()
    st = fn(ctypes.byref(desc), q.data_ptr(), kvq.KVQ_BF16, Hq, lens.data_ptr(), T, 0.0,
            out.data_ptr(), kvq.KVQ_F32, torch.cuda.current_stream().cuda_stream)
    assert st == kvq.KVQ_OK, kvq.kvq_strerror(st)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert torch.equal(out, ref), f"max difference {(out - ref).abs().max().item():.3e}"
    return ref


def test_static_matches_regular_twice():
    fn = _static_fn()
    # A larger shape first, so that the second, smaller call finds the
    # scratch holding stale partials of a different split plan.
    big = _filled_cache(8, 8, 128, 4096, seed=2)
    lens_big = torch.full((8,), 4096, dtype=torch.int32, device="cuda")
    ws_big = kvq.kvq_decode_workspace_bytes(big, 32, 4096)
    assert 0 < ws_big <= STATIC_BYTES
    assert kvq.kvq_decode_split_tokens(big, 32, 4096) < 4096  # several splits per row
    _static_vs_regular(fn, big, 32, lens_big, 4096, seed=7)

    B, Hkv, Hq, D, T = 4, 8, 32, 128, 3000
    cache = _filled_cache(B, Hkv, D, T, seed=1)
    lens = torch.tensor([3000, 1, 1777, 64], dtype=torch.int32, device="cuda")
    ws = kvq.kvq_decode_workspace_bytes(cache, Hq, T)
    assert 0 < ws < ws_big  # this shape uses the scratch too, with another plan
    assert kvq.kvq_decode_split_tokens(cache, Hq, T) < T
    outs = [_static_vs_regular(fn, cache, Hq, lens, T, seed=10 + call) for call in range(2)]
    assert not torch.equal(outs[0], outs[1])  # the two calls had different queries
    assert kvq.kvq_device_error_flags() == 0


def test_static_refuses_shapes_beyond_its_scratch():
    fn = _static_fn()
    # 64 x 128 query heads need 64*128*(128+1)*4 bytes per split: > 4 MiB
    B, Hkv, Hq, D, T = 64, 8, 128, 128, 1024
    cache = kvq.KVCache.allocate(B, Hkv, D, T, 4, 2, 64)
    need = kvq.kvq_decode_workspace_bytes(cache, Hq, T)
    assert need > STATIC_BYTES
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    out = torch.zeros(B, Hq, D, dtype=torch.float32, device="cuda")
    desc = cache.desc()
    st = fn(ctypes.byref(desc), q.data_ptr(), kvq.KVQ_BF16, Hq, lens.data_ptr(), T, 0.0,
            out.data_ptr(), kvq.KVQ_F32, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
