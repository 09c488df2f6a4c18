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
                   ``fused_vs_serial`` and ``fused_vs_attn_only`` are time ratios (fused time
                   divided by the other; below 1 means the fused step is faster);
* ``cpu_baseline`` -- the CPU oracle (fp64, OpenMP) on a bounded sample of the same workload.

``--impl reference`` times that CPU oracle alone (rank 0 only) on the same workload.
``--gpus N`` under torchrun (N > 1, NCCL) runs one Ulysses layer of the workload over the N GPUs
(strong scaling): GPU g computes heads [g*H/N, (g+1)*H/N) and holds the slabs of ranks
[g*P/N, (g+1)*P/N); its fused call stores every finished tile into the slab of the rank
that needs it, on whichever GPU that is (CUDA IPC mappings, NVLink stores), and a
one-element all-reduce after it orders those stores (``multigpu.UlyssesGpu``).  The serial
step is attention, a pack by the exchange kernel, an NCCL all-to-all and an unpack.
When a GPU's Q, K and V fit in L2, every timed step is preceded by a read of a buffer twice
the L2 size, outside the step's events.
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
    ap.add_argument("--dist-backend", choices=["nccl", "gloo"], default="nccl",
                    help="process group for N > 1; gloo orders the GPUs through the host and lets "
                         "several processes share one GPU: a check of the multi-process path, not a "
                         "measurement")
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
    t = torch.tensor([x], dtype=torch.float64, device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda" and dist.get_backend() == "nccl":
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


# The sources that define the attention kernel and its launch (tensor maps, parameters).
KERNEL_SOURCES = ("api.cu", "attn.cu", "ptx.cuh", "xs_internal.cuh")


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":            # string or character literal, copied verbatim
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest() -> str:
    """Hash of the attention kernel's sources, comments and whitespace aside: a profile summary
    is only valid for the kernel it measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ulysses_attention_output_b200", "csrc")
    for fn in KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode() + b"\0" + _code_only(f.read()).encode())
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


def time_steps(fn, steps: int, warmup: int, stream, device, flush=None):
    """Device time (ms) of `steps` calls of fn() on `stream`, max over ranks.

    Without `flush`: one event pair around the back-to-back calls (inputs larger than L2).
    With `flush` (a uint8 device buffer larger than L2): before every call the buffer is
    read on `stream` outside the timed region, so each call starts with no line of its
    inputs in L2; the result is the sum of the calls' own event-pair times."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    if flush is None:
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            fn()
        ev1.record(stream)
        pairs = [(ev0, ev1)]
    else:
        sink = torch.zeros((), dtype=torch.int32, device=device)
        words = flush.view(torch.int32)
        pairs = []
        for _ in range(steps):
            sink.copy_(words.amax())
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            pairs.append((e0, e1))
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    return reduce_max(sum(e0.elapsed_time(e1) for e0, e1 in pairs), device)


def l2_flush_buffer(input_bytes: int, device):
    """A buffer twice the L2 size when the inputs fit in L2, else None (no flush needed)."""
    import torch
    if input_bytes > L2_BYTES:
        return None
    return torch.zeros(2 * L2_BYTES, dtype=torch.uint8, device=device)


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
def workload_config(w, world: int = 1):
    """The `config` object of both arms' lines (the same dict for the same workload and N)."""
    per_gpu = w.qkv_bytes // world
    return {"workload": w.name, "description": w.description, "B": w.B, "H": w.H, "S": w.S,
            "D": w.D, "P": w.P, "structure": w.structure,
            "l2": (f"inputs per GPU larger than L2 ({per_gpu / 2**20:.0f} MiB > 126 MiB), no flush"
                   if per_gpu > L2_BYTES else
                   f"inputs per GPU {per_gpu / 2**20:.0f} MiB fit in L2: a 252 MiB buffer is read "
                   f"before every timed step, outside its events"),
            "parallelism": (f"ulysses{world} (heads {w.H // world} per GPU, NVLink peer stores)"
                            if world > 1 else "single")}


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
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.threads, "kind": "oracle",
                         "sample": smp.describe(n, total / args.steps)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))
    return 0


class SingleGpu:
    """One GPU holds every head and all P slabs: the fused call, its parts and the e2e path."""

    def __init__(self, w, device, stream):
        import torch

        import ulysses_attention_output_b200 as xs
        from ulysses_attention_output_b200 import workloads as W
        self.xs, self.w, self.device, self.stream = xs, w, device, stream
        self.q_h, self.k_h, self.v_h = W.make_inputs(w)
        self.q, self.k, self.v = (t.to(device) for t in (self.q_h, self.k_h, self.v_h))
        self.dest = xs.alloc_dest(w.B, w.H, w.S, w.D, w.P, device=device)
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.flops_gpu = xs.attention_flops(w.B, w.H, w.S, w.D)
        self.input_bytes = w.qkv_bytes

    def fused(self):
        self.xs.attn_a2a_fused(self.q, self.k, self.v, self.dest, stream=self.stream, status=self.status)

    def attn_only(self):
        self.xs.attn(self.q, self.k, self.v, self.out, stream=self.stream, status=self.status)

    def relayout(self):
        self.xs.a2a_relayout(self.out, self.dest, stream=self.stream)

    def serial(self):
        self.attn_only()
        self.relayout()

    def e2e(self):
        """(step function, status tensor, h2d bytes, d2h bytes, extras) through HostPipeline."""
        import torch
        w = self.w
        pipe = self.xs.HostPipeline(w.B, w.H, w.S, w.D, w.P, device=self.device)
        qp, kp, vp = (t.pin_memory() for t in (self.q_h, self.k_h, self.v_h))
        dest_h = [torch.empty(d.shape, dtype=d.dtype).pin_memory() for d in pipe.dest]
        return (lambda: pipe.run(qp, kp, vp, dest_h, stream=self.stream), pipe.status,
                pipe.h2d_bytes, pipe.d2h_bytes, {"head_groups": len(pipe.groups)})

    def close(self):
        pass


class UlyssesGpus:
    """One of N GPUs of a Ulysses layer (NCCL): this GPU's H/N heads; its P/N slabs, which the
    other GPUs' fused calls store into through CUDA IPC mappings over NVLink."""

    def __init__(self, w, device, stream):
        import torch

        import ulysses_attention_output_b200 as xs
        from ulysses_attention_output_b200 import multigpu as MG
        from ulysses_attention_output_b200 import workloads as W
        self.xs, self.w, self.device, self.stream = xs, w, device, stream
        self.layer = MG.UlyssesGpu(w.B, w.H, w.S, w.D, w.P, device=device)
        pl = self.plan = self.layer.plan
        hs = slice(pl.head_offset, pl.head_offset + pl.heads_local)
        self.q_h, self.k_h, self.v_h = (t[:, hs].contiguous() for t in W.make_inputs(w))
        self.q, self.k, self.v = (t.to(device) for t in (self.q_h, self.k_h, self.v_h))
        self.out, self.send, self.recv = self.layer.alloc_exchange_buffers()
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.flops_gpu = xs.attention_flops(w.B, pl.heads_local, w.S, w.D)
        self.input_bytes = 3 * self.q.numel() * 2

    def fused(self):
        self.layer.fused(self.q, self.k, self.v, stream=self.stream, status=self.status)
        self.layer.complete(self.stream)

    def attn_only(self):
        self.xs.attn(self.q, self.k, self.v, self.out, stream=self.stream, status=self.status)

    def relayout(self):
        self.xs.a2a_relayout(self.out, [self.send[r] for r in range(self.w.P)], stream=self.stream)
        self.layer.exchange_packed(self.send, self.recv, stream=self.stream)

    def serial(self):
        self.attn_only()
        self.relayout()

    def e2e(self):
        """Per step through ``LayerHostPipeline``: this GPU's Q, K, V from pinned host memory,
        copied per head group while the fused calls of the groups before run; completion; its
        slabs back to pinned host memory; a second completion so that no GPU's next fused call
        overwrites a slab that is still being copied out."""
        import torch

        from ulysses_attention_output_b200 import multigpu as MG
        pipe = MG.LayerHostPipeline(self.layer)
        qp, kp, vp = (t.pin_memory() for t in (self.q_h, self.k_h, self.v_h))
        slabs_h = torch.empty(self.layer.slabs.shape, dtype=torch.bfloat16).pin_memory()
        return (lambda: pipe.run(qp, kp, vp, slabs_h, stream=self.stream), pipe.status, pipe.h2d_bytes,
                pipe.d2h_bytes, {"head_groups": len(pipe.groups),
                                 "overlap": "input copies of each head group overlap the other groups' "
                                            "kernels; slabs copied out after completion"})

    def close(self):
        self.layer.close()


def run_xs(args):
    import torch
    import torch.distributed as dist

    from ulysses_attention_output_b200 import workloads as W

    rank, local_rank, world = dist_env()
    # gloo may put several processes on one GPU; with NCCL every process has its own GPU
    dev_index = local_rank if args.dist_backend == "nccl" else local_rank % torch.cuda.device_count()
    torch.cuda.set_device(dev_index)
    device = torch.device("cuda", dev_index)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        if args.dist_backend == "nccl":
            dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
        else:
            dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    import ulysses_attention_output_b200 as xs
    xs.load()
    w = W.WORKLOADS[args.workload]
    stream = torch.cuda.Stream(device)
    g = (UlyssesGpus if world > 1 else SingleGpu)(w, device, stream)
    flush = l2_flush_buffer(g.input_bytes, device)

    with torch.cuda.stream(stream):
        with ClockSampler(device.index) as clk:
            fused_ms = time_steps(g.fused, args.steps, args.warmup, stream, device, flush)
        attn_ms = time_steps(g.attn_only, args.steps, args.warmup, stream, device, flush)
        relayout_ms = time_steps(g.relayout, args.steps, args.warmup, stream, device, flush)
        serial_ms = time_steps(g.serial, args.steps, args.warmup, stream, device, flush)
    torch.cuda.synchronize(device)
    if int(g.status.item()) != 0:
        raise RuntimeError(f"device status {int(g.status.item())} after the timed runs")

    flops_job = xs.attention_flops(w.B, w.H, w.S, w.D)   # the whole layer, all GPUs together
    ms_per_step = fused_ms / args.steps
    value = flops_job / (ms_per_step / 1e3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = g.flops_gpu / (ms_per_step / 1e3) / 1e12  # this GPU's launch per step
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    relayout_gbs = 2 * (w.out_bytes // world) / (relayout_ms / args.steps / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        step, st, h2d, d2h, extra = g.e2e()
        n_e2e = max(3, args.steps // 3)
        with torch.cuda.stream(stream):
            e2e_ms = time_steps(step, n_e2e, max(3, args.warmup), stream, device)
        if int(st.item()) != 0:
            raise RuntimeError("device status non-zero in the end-to-end run")
        e2e = {"value": flops_job / (e2e_ms / n_e2e / 1e3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world,
               "ms_per_step": e2e_ms / n_e2e, **extra}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cv, threads, desc = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": cv, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    traffic = profiled_traffic(w.name) if world == 1 else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if world > 1 else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {**workload_config(w, world),
                   **({"dist_backend": "gloo (host-ordered check, not a measurement)"}
                      if world > 1 and args.dist_backend == "gloo" else {})},
        "frac_of_bf16_peak": achieved / peak,
        "serial_ms": serial_ms / args.steps, "attn_only_ms": attn_ms / args.steps,
        "relayout_ms": relayout_ms / args.steps,
        "fused_vs_serial": fused_ms / serial_ms, "fused_vs_attn_only": fused_ms / attn_ms,
        "relayout_gbs": relayout_gbs, "relayout_frac_hbm": relayout_gbs / hbm,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": (f"dram__bytes_read.sum + dram__bytes_write.sum per launch from the "
                                        f"committed ncu summary profiles/attn_fused_{w.name}.md, taken on "
                                        f"kernel sources of the same digest ({source_digest()}); not "
                                        f"measured in this run" if traffic is not None else
                                        "no ncu capture of these kernel sources"),
                     "peak_source": f"{peak_src} bf16 burst", "peak_sustained": peak_sus,
                     "frac_sustained": achieved / peak_sus, "kernel": "attn_fwd_kernel<2,kSeqScatter>"},
        "e2e": e2e, "cpu_baseline": cpu, "clocks": clk.summary(),
        "gpu_launches": args.steps, "impl": "xs",
    }
    g.close()
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
