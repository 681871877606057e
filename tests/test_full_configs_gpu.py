"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times.

Each case builds the benchmark's own step (`bench.Arm`: the same cache shape,
prefill, quantize-append launch, split plan, workspace and output type) for
one configuration (workload and bit pair), runs one step on the GPU, runs the
decode once more with binary32 output, and has the oracle rebuild EVERY
(batch row, kv head) slot from the same seeded inputs (in a pool of `spawn`
processes, one task per slot):

* the whole packed cache (codes and binary16 parameters of every slot) must
  be bit-identical to the oracle's;
* every binary32 output element must be within 2e-3 of the binary64 oracle
  on the oracle's cache (the plain bound);
* every output of the benchmark's own step (bf16 for bf16 workloads) must be
  within 2e-3 plus half an output ulp (its rounding).

The largest binary32 error of each configuration is printed.  The
Qwen/Mistral-shaped configurations also measure attention against
unquantised binary64 attention and check the page's claim that keys-first
(K4V2) beats values-first (K2V4) ("Quantize What Counts", "Results").
"""
import multiprocessing
import os

import numpy as np
import pytest
import torch

import bench
from kv_cache_mixed_kvq_b200 import workloads
from tests.gpu_util import TOL, compare_attention
from tests.oracle_slots import slot_task

pytestmark = pytest.mark.gpu

CASES = [("tiny", (4, 2)), ("llama3_8b", (4, 2)), ("long", (8, 4)), ("long", (4, 2)),
         ("ragged", (4, 2)), ("qwen_mistral", (4, 2)), ("qwen_mistral", (2, 4))]


@pytest.fixture(scope="module")
def pool():
    procs = max(1, min(16, len(os.sched_getaffinity(0))))
    p = multiprocessing.get_context("spawn").Pool(procs)
    yield p
    p.close()
    p.join()


def _bits_of(t):
    return workloads.as_bits(t)


def _row_chunks(arm, w, b, device):
    """The inputs written into batch row b, as (k, v, position) on the CPU:
    the benchmark's prefill (seeded per row) and the step's own append."""
    chunks = []
    if w.name != "llama3_8b":
        kb, vb = workloads.make_kv(w, arm.read[b], seed=100 + b, device=device, batch=1)
        chunks.append((kb[0].cpu(), vb[0].cpu(), 0))
    if arm.n_new:
        s = arm.sets[0]
        chunks.append((s["k"][b].cpu(), s["v"][b].cpu(), arm.pos[b]))
    return chunks


def _slot_arrays(cache):
    """Host copies of the four arrays, one row per (batch row, kv head) slot."""
    slots = cache.batch * cache.kv_heads
    return [t.view(torch.uint8).cpu().numpy().reshape(slots, -1)
            for t in (cache.k_codes, cache.v_codes, cache.k_params, cache.v_params)]


def _run_case(pool, name, bits, dense=False):
    w = workloads.WORKLOADS[name]
    device = torch.device("cuda")
    arm = bench.Arm(w, bits, 1, device)
    arm.step(0)
    torch.cuda.synchronize()
    assert arm.kvq.kvq_device_error_flags() == 0
    s = arm.sets[0]
    out_step = s["out"].clone()
    out32 = arm.kvq.kvq_decode_attention(s["cache"], s["q"], arm.lens, arm.max_len,
                                         out_dtype=torch.float32, workspace=arm.ws)
    torch.cuda.synchronize()
    assert arm.kvq.kvq_device_error_flags() == 0
    gpu = _slot_arrays(s["cache"])
    gq = w.gq
    q_all = s["q"].cpu()

    tasks = []
    for b in range(w.batch):
        chunks = _row_chunks(arm, w, b, device)
        for h in range(w.kv_heads):
            ch = []
            for k, v, pos in chunks:
                kb, dt = _bits_of(k[h])
                vb, _ = _bits_of(v[h])
                ch.append((kb, vb, dt, pos))
            qb, qdt = _bits_of(q_all[b, h * gq:(h + 1) * gq])
            tasks.append({"shape": (w.head_dim, arm.cap, bits[0], bits[1], w.group),
                          "chunks": ch, "q": qb, "q_dtype": qdt, "length": arm.read[b],
                          "max_len": arm.max_len, "dense": dense})
    results = pool.map(slot_task, tasks, chunksize=1)

    names = ("k_codes", "v_codes", "k_params", "v_params")
    ref = np.zeros((w.batch, w.q_heads, w.head_dim), np.float64)
    dense_out = np.zeros_like(ref) if dense else None
    for i, res in enumerate(results):
        b, h = divmod(i, w.kv_heads)
        for name_a, g, o in zip(names, [a[i] for a in gpu], res[:4]):
            if not np.array_equal(g, o):
                bad = np.flatnonzero(g != o)
                raise AssertionError(f"{name} K{bits[0]}V{bits[1]} slot ({b}, {h}) {name_a}: "
                                     f"{bad.size} bytes differ, first at {bad[:8]}")
        assert res[5] == 0
        ref[b, h * gq:(h + 1) * gq] = res[4]
        if dense:
            dense_out[b, h * gq:(h + 1) * gq] = res[6]

    err32 = compare_attention(out32, ref, TOL)  # plain 2e-3 on every element
    err_step = compare_attention(out_step, ref, TOL)
    print(f"{name} K{bits[0]}V{bits[1]}: whole cache bit-exact ({w.batch * w.kv_heads} slots); "
          f"max |error| binary32 out {err32:.2e}, step out ({out_step.dtype}) {err_step:.2e}")
    if dense:
        return float(np.abs(out32.cpu().numpy().astype(np.float64) - dense_out).mean())
    return None


@pytest.mark.parametrize("name,bits", [c for c in CASES if c[0] != "qwen_mistral"])
def test_full_size_workload(pool, name, bits):
    _run_case(pool, name, bits)


def test_qwen_mistral_keys_first_vs_values_first(pool):
    errs = {bits: _run_case(pool, "qwen_mistral", bits, dense=True)
            for bits in ((4, 2), (2, 4))}
    print(f"qwen_mistral mean |error| vs unquantised attention: K4V2 {errs[(4, 2)]:.4e}, "
          f"K2V4 {errs[(2, 4)]:.4e}")
    assert errs[(4, 2)] < errs[(2, 4)]
