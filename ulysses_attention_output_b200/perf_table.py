"""Per-workload timing table of the fused kernel, the serial baseline and their parts, on one GPU.

For each workload (tiny, DiT-XL/2, MMDiT, long, video): the fused call (attention + exchange),
attention alone (head-major output), the exchange pass alone and the serial baseline (the two
in sequence), each the median of ``--reps`` calls timed with CUDA events, with L2 flushed
before every call (a 256 MiB buffer read); TFLOP/s (4 B H S^2 D) and the fraction of the
measured dense bf16 peak; fused / serial and fused / attention-only; the exchange pass in GB/s
(2 B H S D 2 bytes) against the measured copy bandwidth.

Run ``python -m ulysses_attention_output_b200.perf_table`` on a GPU; it prints one JSON object.
``--vendor`` adds, as context only, the cuDNN attention kernel behind torch's
``scaled_dot_product_attention`` (attention alone, no exchange, head-major output) on the same
tensors, timed the same way.
"""
from __future__ import annotations

import argparse
import json
import os
import sys


def _peaks():
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, 6650.0, "fallback"


def measure(name: str, reps: int = 21, warmup: int = 3, vendor: bool = False) -> dict:
    import torch

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import workloads as W
    w = W.WORKLOADS[name]
    q, k, v = (t.cuda() for t in W.make_inputs(w))
    dest = xs.alloc_dest(w.B, w.H, w.S, w.D, w.P, device="cuda")
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    sink = torch.zeros((), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    calls = {
        "fused": lambda: xs.attn_a2a_fused(q, k, v, dest, status=status),
        "attn_only": lambda: xs.attn(q, k, v, out, status=status),
        "relayout": lambda: xs.a2a_relayout(out, dest),
        "serial": lambda: (xs.attn(q, k, v, out, status=status), xs.a2a_relayout(out, dest)),
    }
    if vendor:
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel

        def cudnn_sdpa():
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
                F.scaled_dot_product_attention(q, k, v)
        calls["vendor_cudnn"] = cudnn_sdpa
    samples = {key: [] for key in calls}
    for _ in range(warmup):
        for fn in calls.values():
            fn()
    torch.cuda.synchronize()
    for _ in range(reps):  # the calls alternate, so clock drift affects them alike
        for key, fn in calls.items():
            sink.copy_(flush.view(torch.int32).amax())  # L2 holds clean lines of this buffer only
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record(s)
            fn()
            e1.record(s)
            torch.cuda.synchronize()
            samples[key].append(e0.elapsed_time(e1))
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    med = {key: sorted(vals)[len(vals) // 2] for key, vals in samples.items()}
    peak, peak_sus, hbm, src = _peaks()
    tflops = w.flops / (med["fused"] * 1e-3) / 1e12
    extra = {}
    if vendor:
        extra = {"vendor_cudnn_tflops": w.flops / (med["vendor_cudnn"] * 1e-3) / 1e12,
                 "fused_vs_vendor_cudnn": med["fused"] / med["vendor_cudnn"]}
    return {
        **extra,
        "workload": name, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "P": w.P, "structure": w.structure,
        "reps": reps, "ms": med, "fused_tflops": tflops, "frac_bf16_peak": tflops / peak,
        "frac_bf16_sustained": tflops / peak_sus,
        "attn_only_tflops": w.flops / (med["attn_only"] * 1e-3) / 1e12,
        "fused_vs_serial": med["fused"] / med["serial"], "fused_vs_attn_only": med["fused"] / med["attn_only"],
        "relayout_gbs": 2 * w.out_bytes / (med["relayout"] * 1e-3) / 1e9,
        "relayout_frac_hbm": 2 * w.out_bytes / (med["relayout"] * 1e-3) / 1e9 / hbm,
        "peaks": {"bf16_tflops": peak, "bf16_tflops_sustained": peak_sus, "hbm_gbs": hbm, "source": src},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description="Per-workload timing table (fused, serial, parts)")
    ap.add_argument("--workloads", default="tiny,ditxl,mmdit,long,video")
    ap.add_argument("--reps", type=int, default=21)
    ap.add_argument("--vendor", action="store_true", help="also time cuDNN attention (context)")
    a = ap.parse_args(argv)
    print(json.dumps([measure(n, a.reps, vendor=a.vendor) for n in a.workloads.split(",")]))
    return 0


if __name__ == "__main__":
    sys.exit(main())
