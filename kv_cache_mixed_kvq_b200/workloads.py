"""Seeded synthetic workloads (shapes and value distributions only).

This module holds no quantization or attention arithmetic: it only names the
workload shapes and draws random inputs, and it is the one module that both
the CUDA path's tests/benchmark and the CPU oracle's tests take inputs from.

Shapes follow the models the summary page "Quantize What Counts: More for
Keys, Less for Values" evaluates ("Methodology": Llama-3, Mistral, Phi, Qwen,
DeepSeek; "Results": Qwen3-8B): Llama-3-8B-like (32 query / 8 KV heads,
head_dim 128) and Qwen/Mistral-like (28 / 4) layers.  No dataset or weights
are used; the value distributions below stand in for real activations:

  K[b,h,t,d] = (centre[h,d] + noise[b,h,t,d]) * (10 if d is an outlier channel of h else 1)
  centre ~ N(0, std 2) per (kv head, channel), noise ~ N(0, 1)
  V ~ N(0, 1),  Q ~ N(0, 1)

The per-channel centre and the x10 outlier channels give keys the larger norm
that the page's "Key-Value Norm-Disparity Theorem" predicts (key/value RMS
ratio about 3.9 with 2% outlier channels).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    context: int                      # tokens per sequence (max for ragged)
    dtype: str                        # "f32" or "bf16" for K, V and Q
    bits: tuple                       # ((bits_k, bits_v), ...) variants
    group: int
    outlier_channels: int             # per kv head
    ragged: Optional[tuple] = None    # (lo, hi) inclusive length range
    append: int = 0                   # new tokens quantize-appended per step
    description: str = ""

    @property
    def gq(self) -> int:
        return self.q_heads // self.kv_heads

    def capacity(self) -> int:
        """Positions per slot: context plus appended tokens, rounded up to 16."""
        n = self.context + self.append
        return (n + 15) // 16 * 16


WORKLOADS = {
    "tiny": Workload(
        "tiny", 1, 1, 1, 64, 256, "f32", ((4, 2),), 32, 2,
        description="single head, head_dim 64, 256 tokens, fp32, K4V2 group 32"),
    "llama3_8b": Workload(
        "llama3_8b", 8, 32, 8, 128, 4096, "bf16", ((4, 2),), 64, 3,
        description="Llama-3-8B-shaped decode layer: batch 8, 32q/8kv heads, "
                    "head_dim 128, 4096 tokens, bf16, K4V2 group 64"),
    "long": Workload(
        "long", 1, 32, 8, 128, 32768, "bf16", ((8, 4), (4, 2)), 64, 3, append=1,
        description="long context: batch 1, 32q/8kv, 32768 tokens, K8V4 and K4V2, "
                    "append 1"),
    "ragged": Workload(
        "ragged", 64, 32, 8, 128, 8192, "bf16", ((4, 2),), 64, 3, ragged=(512, 8192),
        description="ragged batch: 64 sequences, lengths uniform in [512, 8192], K4V2"),
    "qwen_mistral": Workload(
        "qwen_mistral", 16, 28, 4, 128, 16384, "bf16", ((4, 2), (2, 4)), 64, 3, append=16,
        description="Qwen/Mistral-shaped: batch 16, 28q/4kv, 16384 tokens, "
                    "K4V2 vs K2V4 at equal budget, append 16"),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def seq_lens(w: Workload, seed: int = 0) -> torch.Tensor:
    """int32 [B] lengths on the CPU (uniform integers in the ragged range)."""
    if w.ragged is None:
        return torch.full((w.batch,), w.context, dtype=torch.int32)
    lo, hi = w.ragged
    g = _generator("cpu", seed)
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def key_channel_profile(kv_heads: int, head_dim: int, outliers: int, seed: int,
                        device="cpu"):
    """(centre [Hkv][D] float32, multiplier [Hkv][D] float32 of 1 or 10)."""
    g = _generator("cpu", seed + 1)
    centre = torch.randn(kv_heads, head_dim, generator=g) * 2.0
    mult = torch.ones(kv_heads, head_dim)
    for h in range(kv_heads):
        idx = torch.randperm(head_dim, generator=g)[:outliers]
        mult[h, idx] = 10.0
    return centre.to(device), mult.to(device)


def make_kv(w: Workload, n_tokens: int, seed: int = 0, device="cpu", dtype: Optional[str] = None,
            batch: Optional[int] = None):
    """K, V of shape [B][Hkv][n_tokens][D] in the workload's dtype on `device`.

    Generated batch row by batch row (bounded temporary memory); the same
    (seed, device) always gives the same tensors.
    """
    dt = TORCH_DTYPE[dtype or w.dtype]
    B = w.batch if batch is None else batch
    centre, mult = key_channel_profile(w.kv_heads, w.head_dim, w.outlier_channels, seed, device)
    g = _generator(device, seed + 2)
    shape = (B, w.kv_heads, n_tokens, w.head_dim)
    k = torch.empty(shape, dtype=dt, device=device)
    v = torch.empty(shape, dtype=dt, device=device)
    for b in range(B):
        noise = torch.randn((w.kv_heads, n_tokens, w.head_dim), generator=g, device=device)
        k[b] = ((centre[:, None, :] + noise) * mult[:, None, :]).to(dt)
        v[b] = torch.randn((w.kv_heads, n_tokens, w.head_dim), generator=g, device=device).to(dt)
        del noise
    return k, v


def make_q(w: Workload, seed: int = 0, device="cpu", dtype: Optional[str] = None,
           batch: Optional[int] = None):
    dt = TORCH_DTYPE[dtype or w.dtype]
    B = w.batch if batch is None else batch
    g = _generator(device, seed + 3)
    return torch.randn((B, w.q_heads, w.head_dim), generator=g, device=device).to(dt)


def as_bits(t: torch.Tensor):
    """numpy view for the oracle: float32 as is, 16-bit types as uint16 bits."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy(), "f32"
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16"), "bf16"
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view("uint16"), "f16"
    raise TypeError(t.dtype)


def make_block_table(lens, capacity: int, page_size: int, seed: int = 0, spare: int = 0):
    """Seeded block table for a paged cache: each row gets ceil(len / P) pages,
    drawn without repetition from a shuffled pool of exactly that many pages
    plus `spare` unused ones (fragmented placement, as after many
    allocations and frees); entries past a row's length are -1.  Returns
    (int32 numpy [len(lens)][capacity / P], num_pages)."""
    import numpy as np

    need = [(int(n) + page_size - 1) // page_size for n in lens]
    num_pages = max(1, sum(need) + spare)
    order = np.random.default_rng(seed).permutation(num_pages)
    table = np.full((len(lens), capacity // page_size), -1, np.int32)
    i = 0
    for b, n in enumerate(need):
        table[b, :n] = order[i:i + n]
        i += n
    return table, num_pages
