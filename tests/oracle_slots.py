"""Oracle work on one (batch row, kv head) slot, run in a process pool.

The full-size parity tests hand every slot of a workload to a pool of
`spawn` processes: each task rebuilds the slot's cache in the CPU oracle from
the same inputs the GPU wrote (bit patterns), and returns the oracle's bytes
and its binary64 attention for the slot's query heads.  Nothing here imports
torch or the CUDA package; no method arithmetic either: every step is an
oracle call.
"""
import numpy as np

import oracle


def slot_task(task):
    """task: dict with
         shape   (D, cap, bits_k, bits_v, group)
         chunks  [(k bits [n][D], v bits [n][D], dtype name, position), ...]
         q       query bit patterns [gq][D], q_dtype
         length  positions attended, max_len (host bound)
         dense   also unquantised attention over the chunks' inputs
       returns (k_codes, v_codes, k_params bytes, v_params bytes, out [gq][D],
                flags, dense out or None)."""
    oracle.build()
    D, cap, bk, bv, G = task["shape"]
    hc = oracle.HostCache(1, 1, D, cap, bk, bv, G)
    for k, v, dt, pos in task["chunks"]:
        flags = hc.quantize_append(k[None, None], v[None, None], [pos], dtype=dt)
        assert flags == 0, f"oracle append flags {flags}"
    q = task["q"][None]
    gq = q.shape[1]
    out, flags = hc.decode_attention(q, gq, [task["length"]], q_dtype=task["q_dtype"],
                                     max_len=task["max_len"])
    dense = None
    if task.get("dense"):
        # unquantised binary64 attention on the same inputs (bit patterns):
        # later chunks overwrite the positions they were written at
        n = task["length"]
        dts = {dt for _, _, dt, _ in task["chunks"]}
        assert len(dts) == 1
        kd = vd = None
        for k, v, dt, pos in task["chunks"]:
            if kd is None:
                kd = np.zeros((n, D), k.dtype)
                vd = np.zeros((n, D), v.dtype)
            m = min(n - pos, k.shape[0])
            kd[pos:pos + m] = k[:m]
            vd[pos:pos + m] = v[:m]
        dense = oracle.attention_dense(kd[None, None], vd[None, None], q, [n],
                                       kv_dtype=dts.pop(), q_dtype=task["q_dtype"])[0]
    return (hc.k_codes, hc.v_codes, hc.k_params.view(np.uint8), hc.v_params.view(np.uint8),
            out[0], flags, dense)
