#!/usr/bin/env python
"""Benchmark: fused DiT attention + Ulysses post-attention All-to-All on B200.

One step = one pass of the hot path over one batch: ``xs_attn_a2a_fused`` on the workload's
Q, K, V (already resident in HBM), writing the P sequence-shard slabs.  Printed as one JSON
line on rank 0:

* ``value``     -- TFLOP/s (4*B*H*S^2*D per step and rank, summed over ranks, divided by the
                   max over ranks of the device time of the K timed steps);
* ``e2e``       -- the same metric through the public API with host buffers
                   (``HostPipeline``): per step, pinned host -> device copies of Q, K, V, the
                   fused calls, device -> host copies of the P slabs, with the heads in groups
                   whose copies overlap the other groups' kernels;
* ``roofline``  -- the fused kernel against the measured dense bf16 tensor peak;
* ``serial_ms`` / ``attn_only_ms`` / ``relayout_ms`` -- attention then the separate exchange
                   pass, attention alone, and the exchange alone, timed the same way;
* ``cpu_baseline`` -- the CPU oracle (fp64, OpenMP) on a bounded sample of the same workload.

``--impl reference`` times that CPU oracle alone (rank 0 only) on the same workload.
``--gpus N`` under torchrun runs N independent replicas (one per GPU): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused attn+A2A TFLOP/s & % BF16 tensor peak; fused vs serial time"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- helpers
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["xs", "reference"], default="xs")
    ap.add_argument("--workload", default="video", help="tiny | ditxl | mmdit | long | video")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU-oracle sample time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_max(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest() -> str:
    """Hash of the CUDA sources: a profile summary is only valid for the kernel it measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ulysses_attention_output_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary, or None when
    the summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", f"attn_fused_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_bytes) or m_sha.group(1) != source_digest():
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        import torch
        ident = str(self.idx)
        try:
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", ident], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        top = max(sm)
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def time_steps(fn, steps: int, warmup: int, stream, device):
    """Device time (ms) of `steps` back-to-back calls of fn() on `stream`, max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    return reduce_max(ev0.elapsed_time(ev1), device)


# ----------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """The CPU oracle on a bounded sample of a workload: the first n sampled query rows of the
    first few heads, each against all S keys of its head (the same seeded values the GPU arm
    uses)."""

    def __init__(self, w, heads: int = 8, max_rows: int = 1024):
        import oracle
        from ulysses_attention_output_b200 import workloads as W
        self.oracle = oracle
        self.w = w
        self.heads = min(w.H, heads)
        q, k, v = W.make_inputs(w)
        sl = (slice(0, 1), slice(0, self.heads))
        self.q, self.k, self.v = (t[sl].contiguous() for t in (q, k, v))
        self.rows = W.sample_rows(w, n=min(w.S, max_rows)).numpy()[:1, :self.heads]
        self.threads = oracle.max_threads()

    def run(self, n: int) -> float:
        t0 = time.perf_counter()
        self.oracle.attention(self.q, self.k, self.v, rows=self.rows[:, :, :n], nthreads=self.threads)
        return time.perf_counter() - t0

    def calibrate(self, target_s: float) -> int:
        """Rows per head so that one run takes about target_s seconds."""
        cap = self.rows.shape[2]
        n = min(cap, max(1, self.threads // self.heads))
        t = self.run(n)
        while t < target_s / 8 and n < cap:
            n = min(cap, n * 4)
            t = self.run(n)
        return min(cap, max(1, int(n * target_s / max(t, 1e-3))))

    def flops(self, n: int) -> float:
        return 4.0 * self.heads * n * self.w.S * self.w.D

    def describe(self, n: int, seconds: float) -> str:
        return (f"{self.heads} heads x {n} query rows (all {self.w.S} keys each) of workload "
                f"'{self.w.name}', fp64, {self.threads} OpenMP threads, {seconds:.1f} s per sample")


def oracle_sample(w, target_s: float):
    """(TFLOP/s, threads, description) of one bounded oracle sample of workload w."""
    smp = OracleSample(w)
    n = smp.calibrate(target_s)
    t = smp.run(n)
    return smp.flops(n) / t / 1e12, smp.threads, smp.describe(n, t)


# ----------------------------------------------------------------------------- arms
def workload_config(w):
    return {"workload": w.name, "description": w.description, "B": w.B, "H": w.H, "S": w.S,
            "D": w.D, "P": w.P, "structure": w.structure,
            "l2": (f"inputs larger than L2 ({w.qkv_bytes / 2**20:.0f} MiB > 126 MiB), no flush"
                   if w.qkv_bytes > L2_BYTES else "L2 flushed between steps")}


def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, bounded samples of the workload."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from ulysses_attention_output_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    smp = OracleSample(w)
    per_step = min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup))
    n = smp.calibrate(per_step)
    for _ in range(args.warmup):
        smp.run(max(1, n // 8))
    times = [smp.run(n) for _ in range(args.steps)]
    total = sum(times)
    value = smp.flops(n) * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.threads, "kind": "oracle",
                         "sample": smp.describe(n, total / args.steps)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))
    return 0


def run_xs(args):
    import torch
    import torch.distributed as dist

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import workloads as W

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    xs.load()
    w = W.WORKLOADS[args.workload]
    B, H, S, D, P = w.B, w.H, w.S, w.D, w.P
    q_h, k_h, v_h = W.make_inputs(w)
    q, k, v = (t.to(device) for t in (q_h, k_h, v_h))
    dest = xs.alloc_dest(B, H, S, D, P, device=device)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    flops = xs.attention_flops(B, H, S, D)

    def fused():
        xs.attn_a2a_fused(q, k, v, dest, stream=stream, status=status)

    def attn_only():
        xs.attn(q, k, v, out, stream=stream, status=status)

    def relayout():
        xs.a2a_relayout(out, dest, stream=stream)

    def serial():
        attn_only()
        relayout()

    with torch.cuda.stream(stream):
        with ClockSampler(device.index) as clk:
            fused_ms = time_steps(fused, args.steps, args.warmup, stream, device)
        attn_ms = time_steps(attn_only, args.steps, args.warmup, stream, device)
        relayout_ms = time_steps(relayout, args.steps, args.warmup, stream, device)
        serial_ms = time_steps(serial, args.steps, args.warmup, stream, device)
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after the timed runs")

    ms_per_step = fused_ms / args.steps
    value = flops * world / (ms_per_step / 1e3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = flops / (ms_per_step / 1e3) / 1e12  # one launch per step on this rank
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    relayout_gbs = 2 * w.out_bytes / (relayout_ms / args.steps / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        pipe = xs.HostPipeline(B, H, S, D, P, device=device)
        qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
        dest_h = [torch.empty(d.shape, dtype=d.dtype).pin_memory() for d in pipe.dest]
        with torch.cuda.stream(stream):
            e2e_ms = time_steps(lambda: pipe.run(qp, kp, vp, dest_h, stream=stream),
                                max(3, args.steps // 3), max(3, args.warmup), stream, device)
        n_e2e = max(3, args.steps // 3)
        if int(pipe.status.item()) != 0:
            raise RuntimeError("device status non-zero in the end-to-end run")
        e2e = {"value": flops * world / (e2e_ms / n_e2e / 1e3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": pipe.h2d_bytes, "d2h_bytes_per_step": pipe.d2h_bytes,
               "ms_per_step": e2e_ms / n_e2e, "head_groups": len(pipe.groups)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cv, threads, desc = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": cv, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(w), "parallelism": f"replicas{world}" if world > 1 else "single"},
        "frac_of_bf16_peak": achieved / peak,
        "serial_ms": serial_ms / args.steps, "attn_only_ms": attn_ms / args.steps,
        "relayout_ms": relayout_ms / args.steps,
        "fused_vs_serial": (serial_ms / fused_ms), "fused_vs_attn_only": fused_ms / attn_ms,
        "relayout_gbs": relayout_gbs, "relayout_frac_hbm": relayout_gbs / hbm,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(w.name),
                     "peak_source": f"{peak_src} bf16 burst", "peak_sustained": peak_sus,
                     "frac_sustained": achieved / peak_sus, "kernel": "attn_fwd_kernel<2,kSeqScatter>"},
        "e2e": e2e, "cpu_baseline": cpu, "clocks": clk.summary(),
        "gpu_launches": args.steps, "impl": "xs",
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_xs(args)


if __name__ == "__main__":
    sys.exit(main())
