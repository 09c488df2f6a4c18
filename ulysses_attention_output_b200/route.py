"""Timing of the Route primitive on one B200: partial attention of routed query rows over each
owner's key/value shard, then the requester's online-softmax merge (page "Move the Query, Not
the Cache: Characterizing Cross-Instance Latent Attention Redistribution Across GPU Fabrics",
"Methodik" -> "Primitiv-Vergleich").

On one GPU the owners' partial attentions run one after another on one stream (each owner
would run its own on its own GPU); the merge follows.  Reported per step:

* ``partial``: time of all owners' partial attentions, TFLOP/s (4 B H Sq S_kv D over the
  sum of the shards) and its fraction of the measured dense bf16 peak;
* ``merge``: time of the merge alone with L2 flushed before it (its inputs come from HBM),
  GB/s over the algorithmic bytes (every part's fp32 O and lse read, bf16 O and fp32 lse
  written) and its fraction of the measured copy bandwidth;
* ``step``: partials + merge back to back (the merge then reads partial results that may
  still be in L2, as it would right after they arrive).

Run ``python -m ulysses_attention_output_b200.route [--workload route] [--steps N]`` on a GPU;
it prints one JSON object.
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
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 6650.0, "fallback"


def measure(name: str = "route", steps: int = 20, warmup: int = 3) -> dict:
    import torch

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import workloads as W
    w = W.ROUTE_WORKLOADS[name]
    q, ks, vs = W.make_route_inputs(w)
    dev = torch.device("cuda")
    qc = q.to(dev)
    kc = [k.to(dev) for k in ks]
    vc = [v.to(dev) for v in vs]
    n = len(w.shards)
    o_parts = [torch.empty(tuple(q.shape), dtype=torch.float32, device=dev) for _ in range(n)]
    l_parts = [torch.empty(tuple(q.shape[:3]), dtype=torch.float32, device=dev) for _ in range(n)]
    out = torch.empty(tuple(q.shape), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(tuple(q.shape[:3]), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def partials():
        for t in range(n):
            xs.attn_partial(qc, kc[t], vc[t], o_parts[t], l_parts[t], stream=stream, status=status)

    def merge():
        xs.lse_merge(o_parts, l_parts, out, lse, stream=stream)

    def timed(fn, flush_l2: bool):
        ms = []
        for i in range(warmup + steps):
            if flush_l2:
                # read 256 MiB: L2 then holds clean lines of this buffer, none of the merge's
                # inputs, and no dirty lines whose write-back would compete with the merge
                flush_sink.copy_(flush.view(torch.int32).amax())
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= warmup:
                ms.append(e0.elapsed_time(e1))
        ms.sort()
        return ms[len(ms) // 2]

    t_partial = timed(partials, False)
    t_merge = timed(merge, True)
    t_step = timed(lambda: (partials(), merge()), False)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    tf_peak, hbm_peak, src = _peaks()
    tflops = w.flops / (t_partial * 1e-3) / 1e12
    gbs = w.merge_bytes / (t_merge * 1e-3) / 1e9
    return {
        "workload": w.name, "description": w.description, "B": w.B, "H": w.H, "Sq": w.Sq,
        "shards": list(w.shards), "D": w.D, "steps": steps, "warmup": warmup,
        "partial": {"ms": t_partial, "tflops": tflops, "frac_bf16_peak": tflops / tf_peak,
                    "flops": w.flops, "launches": n},
        "merge": {"ms": t_merge, "gbs": gbs, "frac_hbm": gbs / hbm_peak, "bytes": w.merge_bytes,
                  "l2": "flushed before each timed merge"},
        "step": {"ms": t_step, "tflops": w.flops / (t_step * 1e-3) / 1e12},
        "peaks": {"bf16_tflops": tf_peak, "hbm_gbs": hbm_peak, "source": src},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description="Route primitive timing (partial attention + merge)")
    ap.add_argument("--workload", default="route")
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)
    print(json.dumps(measure(a.workload, a.steps, a.warmup)))
    return 0


if __name__ == "__main__":
    sys.exit(main())
