"""Wall-clock timing of the CPU oracle on the five workloads (TEST INFRASTRUCTURE: it runs the
oracle, never the product).  Run ``python -m oracle.timing`` on the host of the GPU machine; it
prints one JSON object.

Per workload:
* all host cores (OpenMP default): every query row for the workloads the oracle checks in
  full (tiny, DiT-XL/2, MMDiT), the sampled rows of the parity tests for the long and video
  workloads (256 per head), with the time for every row extrapolated in proportion to the rows;
* one thread: a bounded sample (one head, rows chosen to take about ``--single-seconds``),
  extrapolated to the whole workload in proportion to the query rows (every row costs the same:
  S keys of D dimensions).

Inputs are the seeded workload tensors the GPU arm uses; the FLOP count is 4 B H S^2 D.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import sys
import time

import numpy as np

import oracle


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def time_workload(w, threads: int, single_seconds: float = 5.0):
    """``threads``: the host's default OpenMP thread count, passed explicitly (a one-thread
    run leaves OpenMP set to one thread for later calls that do not name a count)."""
    from ulysses_attention_output_b200 import workloads as W
    q, k, v = W.make_inputs(w)
    full_rows = w.B * w.H * w.S
    out = {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D,
           "flops": float(w.flops), "threads": threads}
    # all cores
    if w.sampled_rows == 0:
        t0 = time.perf_counter()
        oracle.attention(q, k, v, nthreads=threads)
        t = time.perf_counter() - t0
        out.update({"all_cores_rows": full_rows, "all_cores_s": t, "all_cores_full_s": t,
                    "all_cores_extrapolated": False})
    else:
        rows = W.sample_rows(w).numpy()
        n = int(np.prod(rows.shape))
        t0 = time.perf_counter()
        oracle.attention(q, k, v, rows=rows, nthreads=threads)
        t = time.perf_counter() - t0
        out.update({"all_cores_rows": n, "all_cores_s": t, "all_cores_full_s": t * full_rows / n,
                    "all_cores_extrapolated": True})
    # one thread: one head, rows calibrated to about single_seconds
    q1, k1, v1 = (x[:1, :1].contiguous() for x in (q, k, v))
    n = 8
    while True:
        sel = np.arange(min(n, w.S), dtype=np.int32)
        t0 = time.perf_counter()
        oracle.attention(q1, k1, v1, rows=sel, nthreads=1)
        t = time.perf_counter() - t0
        if t > single_seconds / 4 or n >= w.S:
            break
        n = min(w.S, n * 4)
    rows1 = int(min(n, w.S))
    out.update({"single_rows": rows1, "single_s": t, "single_full_s": t * full_rows / rows1})
    out["all_cores_tflops"] = w.flops / out["all_cores_full_s"] / 1e12
    out["single_tflops"] = w.flops / out["single_full_s"] / 1e12
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description="CPU oracle wall-clock timing per workload")
    ap.add_argument("--workloads", default="tiny,ditxl,mmdit,long,video")
    ap.add_argument("--single-seconds", type=float, default=5.0)
    a = ap.parse_args(argv)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from ulysses_attention_output_b200 import workloads as W
    threads = oracle.max_threads()  # before any call sets a count
    res = {"cpu": _cpu_model(), "nproc": os.cpu_count(), "openmp_threads": threads,
           "workloads": [time_workload(W.WORKLOADS[n], threads, a.single_seconds) for n in a.workloads.split(",")]}
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
