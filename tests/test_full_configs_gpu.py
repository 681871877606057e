"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times.

Each case builds the benchmark's own step (`bench.Arm`: the same cache shape,
prefill, quantize-append launch, split plan, workspace and bf16 output) for
one of the five workloads, runs one step on the GPU, and then has the oracle
recompute sampled (batch row, kv head) slots one by one from the same seeded
inputs:

* the slot's packed codes and binary16 parameters must be bit-identical;
* the attention outputs of every query head on that kv head must be within
  2e-3 (plus half a bf16 ulp) of the binary64 oracle on the oracle's cache.

Slots sampled: the first and last slot, the longest and shortest sequence
(ragged lengths) and two seeded random slots.  The Qwen/Mistral-shaped case
also measures both bit splits against unquantised binary64 attention and
checks the page's claim that keys-first (K4V2) beats values-first (K2V4).
"""
import random

import numpy as np
import pytest
import torch

import bench
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, assert_same_cache, compare_attention

pytestmark = pytest.mark.gpu


def _slot_bytes(cache, b, h):
    """The four arrays' bytes of one (batch row, kv head) slot."""
    s = b * cache.kv_heads + h
    out = []
    for t in (cache.k_codes, cache.v_codes, cache.k_params, cache.v_params):
        flat = t.view(torch.uint8).reshape(-1)
        per = flat.numel() // (cache.batch * cache.kv_heads)
        out.append(flat[s * per:(s + 1) * per].cpu().numpy())
    return out


class _OneSlot:
    """Adapter so that assert_same_cache compares one GPU slot with an oracle
    cache of batch 1 and one kv head."""

    def __init__(self, cache, b, h):
        self.k_codes, self.v_codes, self.k_params, self.v_params = [
            torch.from_numpy(x) for x in _slot_bytes(cache, b, h)]


def _slot_inputs(arm, w, b, h, device):
    """The inputs the benchmark wrote into slot (b, h), as (chunks, positions):
    the prefill (other workloads) and the step's own quantize-append."""
    chunks = []
    if w.name != "llama3_8b":
        kb, vb = workloads.make_kv(w, arm.read[b], seed=100 + b, device=device, batch=1)
        chunks.append((kb[:, h:h + 1], vb[:, h:h + 1], 0))
    if arm.n_new:
        s = arm.sets[0]
        chunks.append((s["k"][b:b + 1, h:h + 1], s["v"][b:b + 1, h:h + 1], arm.pos[b]))
    return chunks


def _sampled_slots(w, read):
    rng = random.Random(1234 + len(w.name))
    slots = {(0, 0), (w.batch - 1, w.kv_heads - 1)}
    if w.ragged:
        slots.add((int(np.argmax(read)), 1 % w.kv_heads))
        slots.add((int(np.argmin(read)), 2 % w.kv_heads))
    want = min(6 if w.ragged else 4, w.batch * w.kv_heads)
    while len(slots) < want:
        slots.add((rng.randrange(w.batch), rng.randrange(w.kv_heads)))
    return sorted(slots)


def _check(ora, name, bits, dense_errors=None):
    w = workloads.WORKLOADS[name]
    device = torch.device("cuda")
    arm = bench.Arm(w, bits, 1, device)
    arm.step(0)
    torch.cuda.synchronize()
    assert arm.kvq.kvq_device_error_flags() == 0
    s = arm.sets[0]
    out = s["out"]
    gq = w.gq
    worst = 0.0
    for b, h in _sampled_slots(w, arm.read):
        hc = ora.HostCache(1, 1, w.head_dim, arm.cap, bits[0], bits[1], w.group)
        for k, v, pos in _slot_inputs(arm, w, b, h, device):
            kb, dt = workloads.as_bits(k)
            vb, _ = workloads.as_bits(v)
            assert hc.quantize_append(kb, vb, [pos], dtype=dt) == 0
        assert_same_cache(_OneSlot(arm.sets[0]["cache"], b, h), hc)

        q = s["q"][b:b + 1, h * gq:(h + 1) * gq]
        qb, qdt = workloads.as_bits(q)
        ref, flags = hc.decode_attention(qb, gq, [arm.read[b]], q_dtype=qdt, max_len=arm.max_len)
        assert flags == 0
        got = out[b:b + 1, h * gq:(h + 1) * gq]
        worst = max(worst, compare_attention(got, ref, TOL))

        if dense_errors is not None:
            # unquantised binary64 attention on the same inputs (the last
            # chunk overwrote the prefill's tail positions)
            chunks = _slot_inputs(arm, w, b, h, device)
            kf = chunks[0][0].float().clone()
            vf = chunks[0][1].float().clone()
            for k, v, pos in chunks[1:]:
                kf[:, :, pos:pos + k.shape[2]] = k.float()
                vf[:, :, pos:pos + v.shape[2]] = v.float()
            dense = ora.attention_dense(kf.cpu().numpy(), vf.cpu().numpy(),
                                        q.float().cpu().numpy(), [arm.read[b]])
            dense_errors.append(np.abs(got.float().cpu().numpy() - dense).mean())
    print(f"{name} K{bits[0]}V{bits[1]}: max attention error {worst:.2e} over sampled slots")


@pytest.mark.parametrize("name,bits", [
    ("tiny", (4, 2)),
    ("llama3_8b", (4, 2)),
    ("long", (8, 4)),
    ("long", (4, 2)),
    ("ragged", (4, 2)),
])
def test_full_size_workload(ora, name, bits):
    _check(ora, name, bits)


def test_qwen_mistral_keys_first_vs_values_first(ora):
    errs = {}
    for bits in ((4, 2), (2, 4)):
        e = []
        _check(ora, "qwen_mistral", bits, dense_errors=e)
        errs[bits] = float(np.mean(e))
    print(f"qwen_mistral mean |error| vs unquantised attention: K4V2 {errs[(4, 2)]:.4e}, "
          f"K2V4 {errs[(2, 4)]:.4e}")
    assert errs[(4, 2)] < errs[(2, 4)]
