#!/usr/bin/env python
"""Benchmark of the mixed-precision KV-cache hot path on B200.

The metric is decode attention over the packed cache: the split-K decode
kernel plus the log-sum-exp combine, in algorithmic HBM GB/s (the packed
cache bytes the step must read, plus the query read and the output write)
and KV tokens per second.  Default workload: the ragged batch (64 sequences,
lengths uniform in [512, 8192] from seed 0, 32 query / 8 KV heads,
head_dim 128, K4V2, group 64), the largest configuration, whose step is one
decode step over a resident cache.  Other workloads (`--workload`) time
their own step: the Llama-3-8B-shaped layer quantizes its full cache and then
decodes; the long-context and Qwen/Mistral-shaped layers append their new
tokens and decode.

After the timed region the same JSON line records every configuration
(all workloads and bit pairs) under "configs": the device time of each of
its kernels (median of at least 50 isolated graph replays) with its
algorithmic bytes, GB/s and fraction of the measured HBM copy bandwidth.

Timing: inputs and caches rotate over enough sets that the data touched
between two uses of a set exceeds twice the L2 (the device's own L2 size);
the steps are replayed from a CUDA graph holding one step of every set in
order (consecutive steps chain through programmatic dependent launch, as
consecutive decode calls on a stream do; --step-graphs single replays one
graph per step instead); the timed region is bracketed by a
barrier and a device synchronize, timed with CUDA events on the launch
stream, max over ranks.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--bits K,V] [--group-v G] [--rotate-keys]
                  [--page-size P] [--fused] [--no-configs] [--step-graphs chain|single]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_mixed_kvq_b200 import workloads  # noqa: E402

METRIC = "quantized-KV decode attention HBM GB/s (% of B200 peak) and KV-tokens/s, K4V2"
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "ragged"
# every (workload, bits) configuration, recorded in the "configs" key
# (workload, bits, append fused into the decode call)
CONFIG_SWEEP = (("tiny", (4, 2), False), ("llama3_8b", (4, 2), False), ("long", (8, 4), False),
                ("long", (8, 4), True), ("long", (4, 2), False), ("ragged", (4, 2), False),
                ("qwen_mistral", (4, 2), False), ("qwen_mistral", (4, 2), True),
                ("qwen_mistral", (2, 4), False))
KERNEL_REPS = 60  # isolated graph replays per kernel time (median)


# --------------------------------------------------------------- workload
def step_shape(w: workloads.Workload, bits):
    """Sizes of one step: new tokens written per sequence and lengths read."""
    lens = workloads.seq_lens(w).tolist()
    if w.name == "llama3_8b":
        n_new, pos = w.context, [0] * w.batch          # quantize the full cache
        read = lens
    else:
        n_new = max(w.append, 0)
        pos = [n - n_new for n in lens] if n_new else lens
        read = lens
    return n_new, pos, read


def algorithmic_bytes(w: workloads.Workload, bits, n_new, read_lens, group_v: int = 0):
    """HBM bytes the step must move, by kernel (what the method reads/writes)."""
    bk, bv = bits
    D, G = w.head_dim, w.group
    Gv = group_v or G
    el = 4 if w.dtype == "f32" else 2
    per_tok_cache = D * (bk + bv) // 8 + (D // G) * 4 + (D // Gv) * 4
    rows = w.batch * w.kv_heads * n_new
    quant = rows * (2 * D * el + per_tok_cache) + 4 * w.batch
    tokens = sum(read_lens)
    decode = tokens * w.kv_heads * per_tok_cache + 2 * w.batch * w.q_heads * D * el + 4 * w.batch
    return {"quantize": quant, "decode": decode, "tokens": tokens, "per_token_head": per_tok_cache}


def sha_of(paths):
    """Hash of the code in `paths` (line comments and blank lines removed, so
    that comment-only edits keep recorded counters valid)."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p)) as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "quantize": ["kv_cache_mixed_kvq_b200/csrc/quantize.cuh", "kv_cache_mixed_kvq_b200/csrc/common.cuh"],
    "quantize_rot": ["kv_cache_mixed_kvq_b200/csrc/quantize.cuh",
                     "kv_cache_mixed_kvq_b200/csrc/common.cuh"],
    "decode": ["kv_cache_mixed_kvq_b200/csrc/decode.cuh", "kv_cache_mixed_kvq_b200/csrc/append_rows.cuh",
               "kv_cache_mixed_kvq_b200/csrc/common.cuh"],
    "combine": ["kv_cache_mixed_kvq_b200/csrc/combine.cu", "kv_cache_mixed_kvq_b200/csrc/common.cuh"],
}


def measured_traffic(kernels, workload: str):
    """DRAM bytes per call (sum over `kernels`) from the committed ncu summary
    (profiles/ncu_traffic.json), if every entry still matches its kernel
    source; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    total = 0
    for kernel in kernels:
        rec = data.get(f"{kernel}/{workload}")
        if not rec or rec.get("source_sha") != sha_of(KERNEL_SOURCES[kernel]):
            return None
        total += rec["dram_bytes_per_launch"]
    return total


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return FALLBACK_HBM_GBS, "fallback"


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (one all-reduce; identity at N=1)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 100 ms while the context is open.  With
    window(t0, t1) (host wall-clock seconds), summary() keeps only the
    samples taken inside [t0, t1]: the ones under load."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "timestamp")

    def __init__(self, device_index: int, lead: float = 0.3):
        self.idx = device_index
        self.lead = lead
        self.proc = None
        self.file = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(self.lead)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def window(self, t0: float, t1: float):
        self.t0, self.t1 = t0, t1

    def _in_window(self, row) -> bool:
        if self.t0 is None:
            return True
        try:
            ts = datetime.datetime.strptime(row[9], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except (IndexError, ValueError):
            return False
        return self.t0 <= ts <= self.t1

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return None
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        rows = [[x.strip() for x in r] for r in rows if len(r) >= 9]
        rows = [r for r in rows if self._in_window(r)]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}
        if self.t0 is not None:
            out["window"] = (f"{self.t1 - self.t0:.2f} s: the same steps untimed for 1 s, then "
                             f"the timed region")
        return out


# -------------------------------------------------------------- our arm
class Arm:
    """Device buffers for R rotating sets of inputs + caches, and the step."""

    def __init__(self, w, bits, rotate: int, device, rotate_keys: bool = False,
                 group_v: int = 0, page_size: int = 0, fused: bool = False):
        import kv_cache_mixed_kvq_b200 as kvq
        self.kvq = kvq
        self.w, self.bits = w, bits
        self.n_new, self.pos, self.read = step_shape(w, bits)
        self.cap = w.capacity()
        self.lens = torch.tensor(self.read, dtype=torch.int32, device=device)
        self.max_len = max(self.read)
        self.pos_t = torch.tensor(self.pos, dtype=torch.int32, device=device)
        self.sets = []
        self.page_size = page_size
        # fused: the step's append runs inside the decode call (one launch)
        self.fused = bool(fused) and self.n_new > 0
        if page_size:  # the logical capacity of a paged cache is whole pages
            self.cap = -(-self.cap // page_size) * page_size
        for r in range(rotate):
            paged = {}
            if page_size:
                # a pool of exactly the pages the rows use, shuffled (fragmented)
                need = [max(self.read[b], self.pos[b] + self.n_new) for b in range(w.batch)]
                table, num_pages = workloads.make_block_table(need, self.cap, page_size,
                                                              seed=7 + r)
                paged = dict(page_size=page_size, num_pages=num_pages,
                             block_table=torch.from_numpy(table))
            cache = kvq.KVCache.allocate(w.batch, w.kv_heads, w.head_dim, self.cap, bits[0],
                                         bits[1], w.group, device=device,
                                         rotate_keys=rotate_keys, group_v=group_v, **paged)
            if w.name != "llama3_8b":
                # pre-fill the context (untimed); the step then appends n_new tokens
                for b in range(w.batch):
                    kb, vb = workloads.make_kv(w, self.read[b], seed=100 + r * 1000 + b,
                                               device=device, batch=1)
                    kvq.kvq_quantize_append(_slot_view(cache, b), kb, vb,
                                            torch.zeros(1, dtype=torch.int32, device=device))
            k, v = workloads.make_kv(w, max(self.n_new, 1), seed=r, device=device)
            q = workloads.make_q(w, seed=r, device=device)
            out = torch.empty_like(q)
            self.sets.append(dict(cache=cache, k=k, v=v, q=q, out=out))
        ws = kvq.kvq_decode_workspace_bytes(self.sets[0]["cache"], w.q_heads, self.max_len)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
        self.split_tokens = kvq.kvq_decode_split_tokens(self.sets[0]["cache"], w.q_heads,
                                                        self.max_len)
        # one split per row: the decode writes the output, no combine launch
        self.num_splits = -(-self.max_len // self.split_tokens)

    def quantize(self, r):
        s = self.sets[r]
        if self.n_new and not self.fused:
            self.kvq.kvq_quantize_append(s["cache"], s["k"], s["v"], self.pos_t)

    def decode(self, r):
        s = self.sets[r]
        if self.fused:
            self.kvq.kvq_append_decode_attention(s["cache"], s["k"], s["v"], s["q"], self.lens,
                                                 self.max_len, out=s["out"], workspace=self.ws)
        else:
            self.kvq.kvq_decode_attention(s["cache"], s["q"], self.lens, self.max_len,
                                          out=s["out"], workspace=self.ws)

    def step(self, r):
        self.quantize(r)
        self.decode(r)

    launches_per_step = property(
        lambda self: (1 if self.n_new and not self.fused else 0) +
        (1 if self.num_splits == 1 else 2))


def _slot_view(cache, b):
    """A KVCache over batch row b only (views into the same buffers)."""
    if cache.page_size:  # the whole pool, row b's block table
        return type(cache)(1, cache.kv_heads, cache.head_dim, cache.capacity, cache.bits_k,
                           cache.bits_v, cache.group, cache.k_codes, cache.v_codes,
                           cache.k_params, cache.v_params, rotate_keys=cache.rotate_keys,
                           group_v=cache.group_v, page_size=cache.page_size,
                           num_pages=cache.num_pages,
                           block_table=cache.block_table[b:b + 1].contiguous())
    per = [t.numel() // cache.batch for t in (cache.k_codes, cache.v_codes, cache.k_params,
                                                cache.v_params)]
    return type(cache)(1, cache.kv_heads, cache.head_dim, cache.capacity, cache.bits_k,
                       cache.bits_v, cache.group,
                       *[t[b * n:(b + 1) * n] for t, n in zip(
                           (cache.k_codes, cache.v_codes, cache.k_params, cache.v_params), per)],
                       rotate_keys=cache.rotate_keys, group_v=cache.group_v)


MAX_SETS = 16


def l2_bytes(device) -> int:
    """L2 size of the device, from its properties."""
    return int(torch.cuda.get_device_properties(device).L2_cache_size)


def sets_needed(step_bytes: float, at_least: int, l2: int) -> int:
    """Rotating input/cache sets so that the other sets' data, touched between
    two uses of one set, exceed twice the L2 (at most MAX_SETS; a step whose
    data is far below the L2 then still finds some of it there)."""
    need = 1 + -(-2 * l2 // max(int(step_bytes), 1))
    return max(at_least, min(need, MAX_SETS))


def default_bits(w):
    return w.bits[-1] if w.name == "long" else w.bits[0]


def make_arm(w, bits, device, at_least: int, **kw):
    """An Arm whose rotation exceeds twice the L2, and its algorithmic bytes."""
    n_new0, _, read0 = step_shape(w, bits)
    nb0 = algorithmic_bytes(w, bits, n_new0, read0, kw.get("group_v", 0))
    rotate = sets_needed(nb0["quantize"] * (1 if n_new0 else 0) + nb0["decode"], at_least,
                         l2_bytes(device))
    return Arm(w, bits, rotate, device, **kw), rotate


def roofline_entry(name, ms, kbytes, hbm_peak, peak_kind, traffic, reps):
    ach = kbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(ach / hbm_peak, 4), "traffic": traffic, "ms": round(ms, 5),
            "algorithmic_bytes": kbytes, "timing": f"median of {reps} isolated graph replays",
            "peak_source": f"{peak_kind} hbm_gbs (copy)"}


def kernel_rooflines(arm, w, kern, nbytes, reps, rotate_keys=False):
    """Roofline objects of the step's kernels from their median device times."""
    hbm_peak, peak_kind = peaks()
    roof = {}
    if "quantize" in kern:
        roof["quantize"] = roofline_entry(
            "quantize", kern["quantize"], nbytes["quantize"], hbm_peak, peak_kind,
            measured_traffic(["quantize_rot" if rotate_keys else "quantize"], w.name), reps)
    # the fused call also moves the append's bytes
    kbytes = nbytes["decode"] + (nbytes["quantize"] if arm.fused else 0)
    roof["decode_attention"] = roofline_entry(
        "decode_attention", kern["decode_attention"], kbytes, hbm_peak, peak_kind,
        None if arm.fused else measured_traffic(
            ["decode"] if arm.num_splits == 1 else ["decode", "combine"], w.name), reps)
    roof["decode_attention"]["kernels"] = ("decode (with the append fused)" if arm.fused else
                                           "decode" if arm.num_splits == 1 else
                                           "decode + combine")
    return roof


def timed_replays(steps, rotate, chained):
    """The graph replays of the timed region, in order: None for the graph
    of `rotate` consecutive steps (sets 0 .. rotate-1), r for set r's
    single-step graph.  Exactly `steps` steps, sets taken in turn."""
    if not chained:
        return [i % rotate for i in range(steps)]
    n_chain, rest = divmod(steps, rotate)
    return [None] * n_chain + list(range(rest))


def in_region_roofline(arm, entry, ms_step):
    """When the timed step is the decode-attention call alone (no separate
    quantize launch), its average duration over the timed region is the
    step time: the same roofline from that time, beside the isolated one."""
    if arm.n_new and not arm.fused:
        return {}
    ach = entry["algorithmic_bytes"] / (ms_step / 1e3) / 1e9
    return {"in_timed_region": {
        "achieved": round(ach, 1), "frac": round(ach / entry["peak"], 4), "ms": round(ms_step, 5),
        "timing": "average over the timed steps (each step is this call alone, steps chained "
                  "as consecutive calls on one stream)"}}


def measure_config(name, bits, device, reps, fused=False):
    """Per-kernel device times and rooflines of one configuration's step."""
    w = workloads.WORKLOADS[name]
    arm, rotate = make_arm(w, bits, device, 3, fused=fused)
    for i in range(3):
        arm.step(i % rotate)
    torch.cuda.synchronize()
    kern = per_kernel_times(arm, rotate, reps)
    flags = arm.kvq.kvq_device_error_flags()
    nbytes = algorithmic_bytes(w, bits, arm.n_new, arm.read)
    roof = kernel_rooflines(arm, w, kern, nbytes, reps)
    dec = roof["decode_attention"]
    entry = {
        "workload": name, "bits": f"K{bits[0]}V{bits[1]}",
        "step": step_name(w, arm), "fused_append": arm.fused,
        "step_kernels_ms": round(sum(k["ms"] for k in roof.values()), 5),
        "split_tokens": arm.split_tokens, "num_splits": arm.num_splits,
        "rotating_sets": rotate,
        "kv_tokens": nbytes["tokens"],
        "decode_kv_tokens_per_s": round(nbytes["tokens"] / (dec["ms"] / 1e3), 1),
        "kernels": roof,
        "device_error_flags": flags,
    }
    del arm
    torch.cuda.empty_cache()
    return entry


def step_name(w, arm):
    if w.name == "llama3_8b":
        return "quantize full cache + decode + combine"
    if arm.fused:
        return f"append {arm.n_new} inside the decode + combine"
    if arm.n_new:
        return f"append {arm.n_new} + decode + combine"
    return "decode + combine (one decode step over the resident cache)"


def run_ours(args, rank, world, device):
    w = workloads.WORKLOADS[args.workload]
    bits = tuple(int(x) for x in args.bits.split(",")) if args.bits else default_bits(w)
    arm, rotate = make_arm(w, bits, device, args.rotate, rotate_keys=args.rotate_keys,
                           group_v=args.group_v, page_size=args.page_size, fused=args.fused)
    stream = torch.cuda.current_stream()

    # warm-up (also loads every kernel and the error-word address)
    for i in range(max(args.warmup, 1)):
        arm.step(i % rotate)
    torch.cuda.synchronize()
    flags = arm.kvq.kvq_device_error_flags()
    if flags:
        raise RuntimeError(f"device error flags {flags} during warm-up")

    # one CUDA graph per rotation set, and (--step-graphs chain) one graph of
    # all the sets' steps in order: inside it consecutive steps chain through
    # programmatic dependent launch, as consecutive decode calls on a stream
    # do (each step's kernels still wait for the previous step's to finish
    # before touching memory)
    graphs = []
    for r in range(rotate):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            arm.step(r)
        graphs.append(g)
    chain = None
    if args.step_graphs == "chain" and rotate > 1:
        chain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(chain):
            for r in range(rotate):
                arm.step(r)
        graphs.append(chain)  # (released with the others)
    for i in range(args.warmup):
        graphs[i % rotate].replay()
    if chain is not None:
        chain.replay()
    torch.cuda.synchronize()

    # ---------------- timed region: exactly K steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(physical_index(), lead=0.0) as clocks:
        # the same steps, untimed, for a second before the timed region, so
        # that the clock samples (every 100 ms) are taken under this load:
        # the timed region itself is shorter than one sampling interval
        load_start = time.time()
        while time.time() < load_start + 1.0:
            for g in graphs[:rotate]:
                g.replay()
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for g in timed_replays(args.steps, rotate, chain is not None):
            (chain if g is None else graphs[g]).replay()
        t1.record(stream)
        torch.cuda.synchronize()
        clocks.window(load_start, time.time())
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    ms_step = ms / args.steps
    flags = arm.kvq.kvq_device_error_flags()

    nbytes = algorithmic_bytes(w, bits, arm.n_new, arm.read, args.group_v)
    step_bytes = nbytes["quantize"] * (1 if arm.n_new else 0) + nbytes["decode"]

    # ---------------- per-kernel durations (events inside a graph, GPU kept busy)
    with ClockSampler(physical_index()) as kclocks:
        kern = per_kernel_times(arm, rotate, KERNEL_REPS)
    roof = kernel_rooflines(arm, w, kern, nbytes, KERNEL_REPS, args.rotate_keys)

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(arm, args, step_bytes, world, device)
    graphs.clear()  # release the graphs before any process-group teardown

    probe = read_probe_gbs(device)
    cfg = {
        "workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
        "head_dim": w.head_dim, "context": w.context, "input_dtype": w.dtype,
        "bits_k": bits[0], "bits_v": bits[1], "group": w.group,
        "rotate_keys": bool(args.rotate_keys),
        "group_v": args.group_v or w.group,
        "page_size": args.page_size,
        "fused_append": arm.fused,
        "step": step_name(w, arm),
        "kv_tokens_per_step": nbytes["tokens"],
        "split_tokens": arm.split_tokens,
        "l2": f"{rotate} rotating input/cache sets of {step_bytes / 1e6:.1f} MB (each "
              f"step's data last touched {rotate - 1} steps earlier; L2 "
              f"{l2_bytes(device) / 2**20:.0f} MiB), graph replay"
              + (f" ({rotate} consecutive steps per graph)" if chain is not None
                 else " (one step per graph)"),
        "parallelism": f"replicas{world}" if world > 1 else "single",
    }
    if w.ragged:
        cfg["seq_lens"] = f"uniform in [{w.ragged[0]}, {w.ragged[1]}] from seed 0, " \
                          f"sum {nbytes['tokens']}, max {arm.max_len}"
    result = {
        "metric": METRIC,
        "value": round(world * step_bytes / (ms_step / 1e3) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16-mma/f32",
        "data": "synthetic",
        "config": cfg,
        "kv_tokens_per_s": round(world * nbytes["tokens"] / (ms_step / 1e3), 1),
        # the metric's own kernel(s): decode attention
        "roofline": dict(roof["decode_attention"], kernel="decode_attention",
                         **in_region_roofline(arm, roof["decode_attention"], ms_step)),
        "read_probe": {"value": probe, "unit": "GB/s",
                       "what": "torch sum over 1 GiB fp32, best of 10 (context, not the peak)"},
        "roofline_by_kernel": roof,
        "gpu_launches": arm.launches_per_step * args.steps,
        "device_error_flags": flags,
        "e2e": e2e,
        "clocks": clocks.summary(),
        "clocks_kernel_timing": kclocks.summary(),
        "arith": "binary32 quantizer; exact integer codes as binary16 tensor-core operands "
                 "against binary16 high/low splits of the query and of the output weights, "
                 "binary32 accumulation; binary32 softmax",
    }
    del arm
    torch.cuda.empty_cache()
    if not args.no_configs:
        with ClockSampler(physical_index()) as cclocks:
            result["configs"] = [measure_config(n, b, device, KERNEL_REPS, fused=f)
                                 for n, b, f in CONFIG_SWEEP]
        result["clocks_configs"] = cclocks.summary()
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, bits, args.cpu_seconds)
    return result


def physical_index():
    """nvidia-smi index of the current device."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    cur = torch.cuda.current_device()
    if not vis:
        return cur
    return int(vis.split(",")[cur])


def read_probe_gbs(device, nbytes=1 << 30, reps=10):
    """HBM read bandwidth of a plain reduction over a 1 GiB buffer (torch's
    own kernel, best of `reps`): context for the read-only decode, next to
    the copy bandwidth the roofline divides by."""
    x = torch.ones(nbytes // 4, dtype=torch.float32, device=device)
    x.sum()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    del x
    return round(nbytes / (best / 1e3) / 1e9, 1)


def per_kernel_times(arm, rotate, reps):
    """Median device time of the quantize launch and of the decode-attention
    call (decode + combine) over `reps` replays, from events captured inside
    per-set graphs; a sleep kernel keeps the GPU busy before each replay so
    that launch gaps are not timed."""
    evs, graphs = [], []
    for r in range(rotate):
        e = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e[0].record()
            arm.quantize(r)
            e[1].record()
            arm.decode(r)
            e[2].record()
        evs.append(e)
        graphs.append(g)
    q, d = [], []
    for i in range(reps):
        r = i % rotate
        torch.cuda._sleep(200000)
        graphs[r].replay()
        torch.cuda.synchronize()
        e = evs[r]
        q.append(e[0].elapsed_time(e[1]))
        d.append(e[1].elapsed_time(e[2]))
    out = {"decode_attention": statistics.median(d)}
    if arm.n_new and not arm.fused:
        out["quantize"] = statistics.median(q)
    return out


def run_e2e(arm, args, step_bytes, world, device):
    """Same step through the public API with pinned host buffers: H2D of the
    step's inputs (query, lengths and any new K/V rows), the step's calls,
    D2H of the output, every step.  The cache is the step's resident state.

    The steps are pipelined the way a serving loop would run them: the
    inputs and the output of each step have two device buffers, copies go on
    their own streams, so that step i+1's inputs come in and step i-1's
    output goes out while step i computes; events order every buffer's
    reuse.  The timed region starts before the first copy in and ends after
    the last copy out."""
    s0 = arm.sets[0]
    hk = s0["k"].cpu().pin_memory()
    hv = s0["v"].cpu().pin_memory()
    hq = s0["q"].cpu().pin_memory()
    hlens = arm.lens.cpu().pin_memory()
    hout = [torch.empty_like(s0["out"], device="cpu").pin_memory() for _ in range(2)]
    bufs = [{"k": torch.empty_like(s0["k"]), "v": torch.empty_like(s0["v"]),
             "q": torch.empty_like(s0["q"]), "lens": torch.empty_like(arm.lens),
             "out": torch.empty_like(s0["out"])} for _ in range(2)]
    cache = s0["cache"]
    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()  # noqa: E731  (ordering only)
    in_ready, comp_done, out_done = ([ev(), ev()] for _ in range(3))
    used = [False, False]

    def one(i):
        sl, d = i % 2, bufs[i % 2]
        with torch.cuda.stream(cin):
            if used[sl]:
                cin.wait_event(comp_done[sl])  # step i-2 has read these inputs
            if arm.n_new:
                d["k"].copy_(hk, non_blocking=True)
                d["v"].copy_(hv, non_blocking=True)
            d["q"].copy_(hq, non_blocking=True)
            d["lens"].copy_(hlens, non_blocking=True)
            in_ready[sl].record(cin)
        comp.wait_event(in_ready[sl])
        if used[sl]:
            comp.wait_event(out_done[sl])  # step i-2's output has left
        if arm.fused:
            arm.kvq.kvq_append_decode_attention(cache, d["k"], d["v"], d["q"], d["lens"],
                                                arm.max_len, out=d["out"], workspace=arm.ws,
                                                stream=comp)
        else:
            if arm.n_new:
                arm.kvq.kvq_quantize_append(cache, d["k"], d["v"], arm.pos_t, stream=comp)
            arm.kvq.kvq_decode_attention(cache, d["q"], d["lens"], arm.max_len, out=d["out"],
                                         workspace=arm.ws, stream=comp)
        comp_done[sl].record(comp)
        with torch.cuda.stream(cout):
            cout.wait_event(comp_done[sl])
            hout[sl].copy_(d["out"], non_blocking=True)
            out_done[sl].record(cout)
        used[sl] = True

    def run(n, start=None):
        used[0] = used[1] = False
        if start is not None:
            start.record(comp)
            cin.wait_stream(comp)
        for i in range(n):
            one(i)
        comp.wait_stream(cout)
        comp.wait_stream(cin)

    run(args.warmup)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 20))
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, start=a)
    b.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, device)
    # the last step's output, as copied out, is the step's result
    if not torch.equal(hout[(steps - 1) % 2], bufs[(steps - 1) % 2]["out"].cpu()):
        raise RuntimeError("e2e: the output copied out differs from the device output")
    h2d = hq.numel() * hq.element_size() + hlens.numel() * hlens.element_size()
    if arm.n_new:
        h2d += hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    return {"value": round(world * step_bytes / (ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hout[0].numel() * hout[0].element_size(),
            "what": "the same step through the public API: pinned host query and lengths "
                    "(and new K/V rows when the step appends) copied in, the output copied "
                    "out, every step, double-buffered on copy streams so that the copies "
                    "overlap the neighbouring steps' kernels; the cache stays resident on "
                    "the device"}


# ---------------------------------------------------------- oracle (CPU)
def step_quantizes(w) -> bool:
    """Whether the workload's step runs the quantizer (else it only decodes)."""
    return w.name == "llama3_8b" or w.append > 0


def row_bytes(w, bits, length):
    """Algorithmic bytes of one batch row of `length` tokens: (quantize of its
    whole context, decode of all its query heads)."""
    bk, bv = bits
    D, G = w.head_dim, w.group
    el = 4 if w.dtype == "f32" else 2
    per_tok = D * (bk + bv) // 8 + 2 * (D // G) * 4
    quant = w.kv_heads * length * (2 * D * el + per_tok) + 4
    decode = length * w.kv_heads * per_tok + 2 * w.q_heads * D * el + 4
    return quant, decode


class OracleRow:
    """One batch row of the workload prepared for the oracle: its inputs
    (bit patterns) and, for decode-only steps, its cache already quantized
    (untimed: the step reads a resident cache)."""

    def __init__(self, w, bits, row, seed):
        import oracle
        self.w, self.bits = w, bits
        self.length = int(workloads.seq_lens(w)[row % w.batch])
        ks, vs = workloads.make_kv(w, self.length, seed=seed, batch=1)
        q = workloads.make_q(w, seed=seed, batch=1)
        self.kb, self.dt = workloads.as_bits(ks)
        self.vb, _ = workloads.as_bits(vs)
        self.qb, _ = workloads.as_bits(q)
        self.cap = (self.length + 15) // 16 * 16
        self.hc = None
        if not step_quantizes(w):
            self.hc = self._quantized(oracle)

    def _quantized(self, oracle):
        w, bits = self.w, self.bits
        hc = oracle.HostCache(1, w.kv_heads, w.head_dim, self.cap, bits[0], bits[1], w.group)
        hc.quantize_append(self.kb, self.vb, [0], dtype=self.dt)
        return hc

    def run(self):
        """One timed oracle pass: (quantize s, decode s, quantize bytes, decode
        bytes, KV tokens).  Decode-only steps time the decode alone."""
        import oracle
        tq, bq = 0.0, 0
        hc = self.hc
        if hc is None:
            t0 = time.perf_counter()
            hc = self._quantized(oracle)
            tq = time.perf_counter() - t0
            bq = row_bytes(self.w, self.bits, self.length)[0]
        t1 = time.perf_counter()
        hc.decode_attention(self.qb, self.w.q_heads, [self.length], q_dtype=self.dt)
        td = time.perf_counter() - t1
        return tq, td, bq, row_bytes(self.w, self.bits, self.length)[1], self.length


_POOL_ROW = None


def _oracle_init(name, bits):
    """Pool worker set-up: one batch row (index and seed from the worker's
    pid, so that workers cover the workload's length mix), prepared before
    any timed task."""
    global _POOL_ROW
    w = workloads.WORKLOADS[name]
    _POOL_ROW = OracleRow(w, bits, os.getpid(), seed=os.getpid() % 1000)


def _oracle_row(_):
    """Pool worker: one single-row oracle pass on the worker's row."""
    return _POOL_ROW.run()


MAX_ORACLE_PROCS = 16  # each worker process imports torch: bounded host memory and start-up


def host_cores() -> int:
    """Host cores the oracle pool uses: the cores this process may run on, at
    most MAX_ORACLE_PROCS."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, MAX_ORACLE_PROCS))


class OraclePool:
    """Single-row oracle passes on every host core: one process per core,
    started with `spawn` (never forked from a process that has used CUDA)."""

    def __init__(self, procs: int, w, bits):
        import multiprocessing
        self.procs = procs
        self.pool = multiprocessing.get_context("spawn").Pool(
            procs, initializer=_oracle_init, initargs=(w.name, bits))

    def run(self, rows: int):
        """Wall seconds and summed results of `rows` single-row passes."""
        t = time.perf_counter()
        res = self.pool.map(_oracle_row, range(rows), chunksize=1)
        wall = time.perf_counter() - t
        return wall, [sum(r[i] for r in res) for i in range(5)]

    def close(self):
        self.pool.close()
        self.pool.join()


def what_sample(w):
    return ("quantize its full context + decode all its query heads" if step_quantizes(w) else
            "decode all its query heads over its resident quantized cache")


def cpu_baseline(w, bits, budget_s):
    """The oracle on the host's cores: single-threaded (quantize and decode
    timed separately) for about budget_s / 2, then one row per process on
    every core for about budget_s / 2 of wall time (the reported value)."""
    import oracle
    oracle.build()
    sq = sd = bq = bd = 0.0
    toks, runs = 0, 0
    while sq + sd < budget_s / 2 or runs == 0:
        a, b, c, d, t = OracleRow(w, bits, runs, seed=runs).run()
        sq, sd, bq, bd, toks, runs = sq + a, sd + b, bq + c, bd + d, toks + t, runs + 1
    single = {"value": round((bq + bd) / (sq + sd) / 1e9, 4), "unit": "GB/s", "cores": 1,
              "decode_gbs": round(bd / sd / 1e9, 4),
              "kv_tokens_per_s": round(toks / (sq + sd), 1),
              "sample": f"{runs} x one batch row of {w.name}, {sq + sd:.1f} s"}
    if sq > 0:
        single["quantize_gbs"] = round(bq / sq / 1e9, 4)
    procs = host_cores()
    out = {"value": single["value"], "unit": "GB/s", "cores": 1, "kind": "oracle",
           "kv_tokens_per_s": single["kv_tokens_per_s"],
           "sample": f"{runs} x one batch row of {w.name} ({what_sample(w)}), "
                     f"single-threaded C oracle, {sq + sd:.1f} s",
           "single_thread": single}
    if procs > 1:
        per_row = (sq + sd) / runs
        rows = procs * max(1, int(round(budget_s / 2 / per_row)))  # ~budget_s / 2 of wall
        pool = OraclePool(procs, w, bits)
        try:
            pool.run(procs)  # start-up (imports, inputs) outside the timing
            wall, (_, _, pb_q, pb_d, ptoks) = pool.run(rows)
        finally:
            pool.close()
        out.update({"value": round((pb_q + pb_d) / wall / 1e9, 4), "cores": procs,
                    "kv_tokens_per_s": round(ptoks / wall, 1),
                    "sample": f"{rows} x one batch row of {w.name} ({what_sample(w)}), C "
                              f"oracle, one process per core on {procs} cores, {wall:.1f} s "
                              f"wall"})
    return out


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on a bounded sample per step:
    one batch row per host core (one process per core)."""
    import oracle
    oracle.build()
    w = workloads.WORKLOADS[args.workload]
    bits = tuple(int(x) for x in args.bits.split(",")) if args.bits else default_bits(w)
    procs = host_cores()
    pool = OraclePool(procs, w, bits)
    try:
        for i in range(args.warmup):
            pool.run(procs)
        tot_s, tot_b, tot_t = 0.0, 0.0, 0
        for i in range(args.steps):
            wall, (_, _, bq, bd, t) = pool.run(procs)
            tot_s, tot_b, tot_t = tot_s + wall, tot_b + bq + bd, tot_t + t
    finally:
        pool.close()
    value = round(tot_b / tot_s / 1e9, 4)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads,
                   "kv_heads": w.kv_heads, "head_dim": w.head_dim, "context": w.context,
                   "bits_k": bits[0], "bits_v": bits[1], "group": w.group,
                   "step": f"{procs} batch rows of the workload per step, one per host core, "
                           f"each: {what_sample(w)} (bounded sample)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": procs, "kind": "oracle",
                         "sample": f"{procs} batch rows per step ({what_sample(w)}), C "
                                   f"oracle, one process per core"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "kv_tokens_per_s": round(tot_t / tot_s, 1),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--step-graphs", choices=["chain", "single"], default="chain",
                    help="timed steps replayed from one graph per rotating set (single) or "
                         "from one graph holding every set's step in order (chain)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--bits", default=None, help="bits_k,bits_v (default: the workload's)")
    ap.add_argument("--rotate", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration kernel times after the timed region")
    ap.add_argument("--group-v", type=int, default=0,
                    help="values' group size (default: the workload's group)")
    ap.add_argument("--fused", action="store_true",
                    help="append inside the decode call (kvq_append_decode_attention)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="paged cache layout with pages of this many positions (0: slots)")
    ap.add_argument("--rotate-keys", action="store_true",
                    help="cache with key-only Walsh-Hadamard rotation (KVQ_FLAG_ROTATE_KEYS)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        res = run_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
