"""Host-side logic of the benchmark, on the CPU: the algorithmic byte counts
behind every GB/s figure, the max-over-ranks reduction of the timed region
(world size 2 over gloo), and the reference arm's launch under torchrun
(rank 0 alone prints one JSON line, the other rank exits 0)."""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kv_cache_mixed_kvq_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_llama_layer():
    w = workloads.WORKLOADS["llama3_8b"]
    n_new, pos, read = bench.step_shape(w, (4, 2))
    assert n_new == 4096 and pos == [0] * 8 and read == [4096] * 8
    nb = bench.algorithmic_bytes(w, (4, 2), n_new, read)
    # per token-head: 128*(4+2)/8 code bytes + 2 groups * (scale, zero) binary16
    assert nb["per_token_head"] == 96 + 16
    rows = 8 * 8 * 4096
    # quantize: bf16 K and V read, packed cache written, positions read
    assert nb["quantize"] == rows * (2 * 128 * 2 + 112) + 4 * 8 == 163_577_888
    # decode: every cached token-head once, bf16 Q read and output written, lengths
    assert nb["decode"] == 8 * 4096 * 8 * 112 + 2 * 8 * 32 * 128 * 2 + 4 * 8 == 29_491_232


def test_step_shapes_append_workloads():
    for name, n in (("long", 1), ("qwen_mistral", 16), ("ragged", 0), ("tiny", 0)):
        w = workloads.WORKLOADS[name]
        n_new, pos, read = bench.step_shape(w, w.bits[0])
        assert n_new == n
        lens = workloads.seq_lens(w).tolist()
        assert read == lens
        assert pos == ([x - n for x in lens] if n else lens)
        assert max(read) <= w.capacity()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["value"] > 0 and res["unit"] == "GB/s"
    assert res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_baseline_uses_every_core():
    import bench
    w = bench.workloads.WORKLOADS["tiny"]
    res = bench.cpu_baseline(w, w.bits[0], 0.5)
    assert res["kind"] == "oracle" and res["value"] > 0
    assert res["cores"] == bench.host_cores()
    single = res["single_thread"]
    # the tiny step decodes a resident cache: only the decode is timed
    assert single["cores"] == 1 and single["decode_gbs"] > 0 and "quantize_gbs" not in single


def test_oracle_row_times_the_phases_of_the_step():
    import bench
    w = bench.workloads.WORKLOADS["llama3_8b"]  # its step quantizes the full cache
    tq, td, bq, bd, toks = bench.OracleRow(w, (4, 2), 0, seed=0).run()
    assert tq > 0 and td > 0 and toks == 4096
    assert (bq, bd) == bench.row_bytes(w, (4, 2), 4096)
    # one row's share of the whole step's algorithmic bytes
    nb = bench.algorithmic_bytes(w, (4, 2), 4096, [4096] * 8)
    assert bq * 8 == nb["quantize"] and bd * 8 == nb["decode"]
    w = bench.workloads.WORKLOADS["ragged"]  # decode only, over a quantized row
    row = bench.OracleRow(w, (4, 2), 5, seed=1)
    assert row.length == int(bench.workloads.seq_lens(w)[5]) and row.hc is not None


def test_rotation_exceeds_twice_the_l2():
    import bench
    l2 = 126 * 2**20
    for step_bytes in (1e3, 29.4e6, 118e6, 193e6, 248e6, 1e9):
        n = bench.sets_needed(step_bytes, 3, l2)
        assert 3 <= n <= bench.MAX_SETS
        if n < bench.MAX_SETS:
            assert (n - 1) * step_bytes >= 2 * l2
    assert bench.sets_needed(248e6, 3, l2) == 3      # the ragged step keeps three sets
    assert bench.sets_needed(29.4e6, 3, l2) == 10


def test_config_sweep_covers_every_workload_and_bit_pair():
    import bench
    got = {(n, b) for n, b, _ in bench.CONFIG_SWEEP}
    want = {(n, b) for n, w in bench.workloads.WORKLOADS.items() for b in w.bits}
    assert got == want
    # the fused append is measured beside the two-call step of every workload
    # that appends during decode
    fused = {n for n, _, f in bench.CONFIG_SWEEP if f}
    appending = {n for n, w in bench.workloads.WORKLOADS.items() if w.append > 0}
    assert fused == appending
    assert bench.DEFAULT_WORKLOAD == "ragged" and bench.KERNEL_REPS >= 50


def test_clock_summary_keeps_only_samples_inside_the_window(tmp_path):
    # nvidia-smi rows (csv, no header, no units): index, sm clock, max clock,
    # power, active reasons, four reason flags, timestamp
    def row(t, mhz, cap="Not Active"):
        ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"0, {mhz}, 1965, 600.0, 0x0, Not Active, Not Active, Not Active, {cap}, {ts}"

    t = 1_800_000_000.0
    f = open(tmp_path / "clocks.csv", "w+")
    f.write("\n".join([row(t - 0.5, 900), row(t + 0.1, 1965), row(t + 0.2, 1950, "Active"),
                       row(t + 2.0, 1000)]) + "\n")
    s = bench.ClockSampler(0, lead=0.0)
    s.proc, s.file = object(), f
    s.window(t, t + 1.0)
    out = s.summary()
    assert out["samples"] == 2
    assert out["sm_mhz"] == (1965 + 1950) / 2
    assert out["reasons"] == ["sw_power_cap"]
    s.t0 = None  # no window: every sample
    assert s.summary()["samples"] == 4


def test_timed_replays_run_exactly_k_steps_in_set_order():
    for rotate in (1, 2, 3, 5):
        for steps in (1, 2, 3, 7, 50):
            for chained in (False, True):
                order = []
                for g in bench.timed_replays(steps, rotate, chained and rotate > 1):
                    order.extend(range(rotate) if g is None else [g])
                assert len(order) == steps
                assert order == [i % rotate for i in range(steps)]
