"""Burst-Gap characterisation of store bursts on one B200.

The Burst-Gap model of the X-Stage paper (explainer page, "Technisches Resuemee" ->
"Methodik: Die X-Stage-Abstraktion und das Burst-Gap-Modell") gives the sender-visible issue
time of a burst of aggregate volume V issued by K producers that compute for a gap G between
bursts as

    T_iss(G; K, V) = max(T0_iss(K, V), V / R - G)

with T0_iss the backpressure-free issue time, R the effective drain rate and Q the effective
outstanding capacity (the volume that can be in flight before issue stalls).  The pages give
the model and its parameters by name only (R of about 717 GB/s on their remote-store path; no
T0_iss or Q values).

This module measures T_iss with the ``xs_burst_probe`` kernel (16-byte stores into a scratch
ring in this GPU's memory, i.e. the local stand-in for remote stores) over a grid of
(K, V, G), and fits the three parameters:

* T0_iss(K, V): the issue time at the largest gaps, where every earlier burst has drained;
* R: 1 / slope of T_iss against V at G = 0 over the volumes in the drain-dominated regime
  (issue time more than 25% above the backpressure-free time);
* Q: the knee -- the largest volume at G = 0 whose issue time is still within 25% of the
  backpressure-free time at that volume.

``predict`` evaluates the model; ``completion_coupled`` is the counter-model in which the
issuer waits until its stores have drained (issue time V / R for every burst, no overlap).

Run ``python -m ulysses_attention_output_b200.burst_gap [--large] [--wide] [--fused] [--spans]``
or ``--knee`` on a GPU for a sweep (``--large``: bursts of 4..64 MB from 148 producers;
``--knee``: G swept densely through the knee at 32..128 MiB with one volume held out and
predicted from the others' fit, plus drained single bursts up to 512 MiB for the outstanding
capacity Q; ``--wide``: 1024
threads per producer; ``--fused``: also time the fused kernel against attention alone on the
MMDiT, long and video workloads and set the measured overhead beside both models'
predictions; ``--spans``: the per-tile store-issue span histogram of the fused kernel,
recorded by ``xs_attn_a2a_fused_spans``, beside both models' predictions); it prints one JSON
object with the raw points and the fit.
"""
from __future__ import annotations

import json
import math
import sys

import numpy as np


# ----------------------------------------------------------------------------- model
def predict(t0_ns: float, r_gbs: float, volume_bytes: float, gap_ns: float) -> float:
    """Burst-Gap model: sender-visible issue time (ns) of one burst."""
    return max(t0_ns, volume_bytes / r_gbs - gap_ns)


def completion_coupled(r_gbs: float, volume_bytes: float) -> float:
    """Counter-model: the issuer waits for its burst to drain before it resumes (ns)."""
    return volume_bytes / r_gbs


# ----------------------------------------------------------------------------- measurement
def issue_times_ns(stamps: np.ndarray, drop: int = 8):
    """Per-burst sender-visible issue times (ns) from the probe's stamps [K, N, 4].

    Cycles are converted with the SM clock rate measured from the same stamps (clock64 and
    global-timer deltas between the first kept burst and the last one of each producer).
    Returns (issue_ns [K, N-drop], gap_ns [K, N-drop], clock_ghz).
    """
    st = np.asarray(stamps, dtype=np.int64)
    k, n, _ = st.shape
    if n - drop < 2:
        raise ValueError("need at least two bursts after the dropped ones")
    kept = st[:, drop:, :]
    d_clk = (kept[:, -1, 0] - kept[:, 0, 0]).astype(np.float64)
    d_ns = (kept[:, -1, 3] - kept[:, 0, 3]).astype(np.float64)
    ok = d_ns > 0
    ghz = float(np.median(d_clk[ok] / d_ns[ok])) if ok.any() else float("nan")
    issue = (kept[:, :, 1] - kept[:, :, 0]) / ghz
    gap = (kept[:, :, 2] - kept[:, :, 1]) / ghz
    return issue, gap, ghz


def run_point(xs, torch, scratch, producers: int, volume: int, gap_cycles: int, n_bursts: int,
              threads: int = 256, drop: int = 8):
    stamps = torch.zeros((producers, n_bursts, 4), dtype=torch.int64, device=scratch.device)
    xs.burst_probe(scratch, stamps, burst_bytes=volume, producers=producers, gap_cycles=gap_cycles,
                   n_bursts=n_bursts, threads_per_producer=threads)
    torch.cuda.synchronize()
    issue, gap, ghz = issue_times_ns(stamps.cpu().numpy(), drop)
    return {"K": producers, "V": volume, "G_cycles": gap_cycles, "G_ns": float(np.median(gap)),
            "t_iss_ns": float(np.median(issue)), "t_iss_p90_ns": float(np.percentile(issue, 90)),
            "clock_ghz": ghz}


def sweep(volumes, producers, gaps, n_bursts: int = 64, drop: int = 8,
          scratch_bytes: int = 1 << 30, threads: int = 256):
    """Measure T_iss over the (K, V, G) grid.  Volumes are per burst over all producers."""
    import torch

    import ulysses_attention_output_b200 as xs
    scratch = torch.empty(scratch_bytes, dtype=torch.uint8, device="cuda")
    out = []
    for k in producers:
        for v in volumes:
            vv = (v // (16 * k)) * 16 * k
            if vv <= 0:
                continue
            for g in gaps:
                out.append(run_point(xs, torch, scratch, k, vv, g, n_bursts, threads, drop))
    return out


# ----------------------------------------------------------------------------- fit
def fit(points, knee_tolerance: float = 0.25):
    """Fit T0_iss(K, V), R and Q from sweep points (dicts with K, V, G_ns, t_iss_ns)."""
    by_kv = {}
    for p in points:
        by_kv.setdefault((p["K"], p["V"]), []).append(p)
    t0 = {}
    for (k, v), pts in by_kv.items():
        gmax = max(q["G_ns"] for q in pts)
        floor = [q["t_iss_ns"] for q in pts if q["G_ns"] >= 0.5 * gmax]
        t0[(k, v)] = float(min(floor))
    kmax = max(k for k, _ in by_kv)
    zero_gap = sorted(((v, min(q["t_iss_ns"] for q in pts if q["G_ns"] == min(x["G_ns"] for x in pts)))
                       for (k, v), pts in by_kv.items() if k == kmax))
    vols = np.array([v for v, _ in zero_gap], dtype=np.float64)
    times = np.array([t for _, t in zero_gap], dtype=np.float64)
    knee = None
    for v, t in zero_gap:
        if t <= (1.0 + knee_tolerance) * t0[(kmax, int(v))]:
            knee = int(v)
    # drain-dominated points: issue time at G = 0 clearly above the backpressure-free time
    drain = np.array([t > (1.0 + knee_tolerance) * t0[(kmax, int(v))] for v, t in zero_gap])
    if drain.sum() < 2:
        drain = vols >= np.sort(vols)[-3]
    slope, intercept = np.polyfit(vols[drain], times[drain], 1)
    r_gbs = 1.0 / slope if slope > 0 else float("inf")
    return {"T0_ns": {f"K={k},V={v}": val for (k, v), val in sorted(t0.items())},
            "R_GBps": float(r_gbs), "intercept_ns": float(intercept), "Q_bytes": knee,
            "K_for_R": kmax}


def t0_at(points, k: int, volume: float) -> float:
    """Backpressure-free issue time at (k, volume), linear in V between / beyond the two
    nearest swept volumes of the largest gaps."""
    f = fit([p for p in points if p["K"] == k])
    vols = sorted(int(key.split("V=")[1]) for key in f["T0_ns"])
    t = [f["T0_ns"][f"K={k},V={v}"] for v in vols]
    if volume <= vols[0]:
        return t[0]
    i = max(j for j in range(len(vols) - 1) if vols[j] <= volume) if volume < vols[-1] else len(vols) - 2
    return t[i] + (t[i + 1] - t[i]) * (volume - vols[i]) / (vols[i + 1] - vols[i])


def epilogue_models(points, n_ctas: int, bytes_per_cta: int, gap_ns: float):
    """Sender-visible time of one wave of fused epilogues (n_ctas CTAs each storing
    bytes_per_cta, then a compute gap gap_ns before the next wave): the Burst-Gap prediction
    max(T0_iss, V/R - G) and the completion-coupled one (the issuer waits V/R)."""
    f = fit(points)
    v = n_ctas * bytes_per_cta
    t0 = t0_at(points, f["K_for_R"], v)
    return {"V_bytes": v, "T0_ns": t0, "burst_gap_ns": predict(t0, f["R_GBps"], v, gap_ns),
            "completion_coupled_ns": max(t0, completion_coupled(f["R_GBps"], v))}


def fused_overhead_check(points, names=("mmdit", "long", "video"), reps: int = 15):
    """Measured fused-minus-attention-only time against the two models, per workload."""
    import torch

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import workloads as W
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = []
    for name in names:
        w = W.WORKLOADS[name]
        g = torch.Generator(device="cuda").manual_seed(0)
        q, k, v = (torch.randn(w.shape(), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        dest = xs.alloc_dest(w.B, w.H, w.S, w.D, w.P, device="cuda")
        o = torch.empty_like(q)
        # Alternate the two kernels call by call and take per-call medians, so that clock
        # drift under the power cap affects both alike.
        fns = {"fused": lambda: xs.attn_a2a_fused(q, k, v, dest), "attn_only": lambda: xs.attn(q, k, v, o)}
        samples = {label: [] for label in fns}
        for _ in range(3):
            for fn in fns.values():
                fn()
        torch.cuda.synchronize()
        for _ in range(reps):
            for label, fn in fns.items():
                e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                samples[label].append(e0.elapsed_time(e1) * 1e6)  # ns
        times = {label: float(np.median(v)) for label, v in samples.items()}
        n_items = w.B * w.H * ((w.S + 255) // 256)
        waves = math.ceil(n_items / sms)
        item_ns = times["attn_only"] / waves
        m = epilogue_models(points, sms, 2 * 128 * w.D * 2, item_ns)
        out.append({"workload": name, "S": w.S, "fused_ns": times["fused"],
                    "attn_only_ns": times["attn_only"],
                    "measured_overhead_ns": times["fused"] - times["attn_only"],
                    "waves": waves, "item_ns": item_ns,
                    "pred_burst_gap_exposed_ns": waves * max(0.0, m["burst_gap_ns"] - m["T0_ns"]),
                    "pred_completion_coupled_exposed_ns": waves * m["completion_coupled_ns"],
                    "model": m})
        del q, k, v, dest, o
    return out


def span_stats(spans, grid: int, ghz: float | None = None, bins: int = 30):
    """Per-tile store-issue spans from the stamps of ``xs_attn_a2a_fused_spans``.

    spans: [n_items, 2, 4, 3] (SM clock before the first store, SM clock after the last
    store issue, global timer ns), items striped over ``grid`` CTAs (item i on CTA i % grid).
    A tile's span runs from the earliest of its four warps' first stamps to the latest of
    their second stamps (one SM clock).  The SM clock rate is taken from the stamps of CTAs
    that ran several items (clock and timer deltas between their first and last item) unless
    ``ghz`` is given.  The gap is the time from a tile's last store issue to the first store
    of the next item's same tile on the same CTA (the compute gap G between its bursts).
    """
    st = np.asarray(spans, dtype=np.int64)
    n = st.shape[0]
    start = st[:, :, :, 0].min(axis=2)
    end = st[:, :, :, 1].max(axis=2)
    cyc = (end - start).astype(np.float64)            # [n_items, 2]
    if ghz is None:
        rates = []
        for c in range(min(grid, n)):
            items = np.arange(c, n, grid)
            if len(items) < 2:
                continue
            d_clk = st[items[-1], 0, 0, 0] - st[items[0], 0, 0, 0]
            d_ns = st[items[-1], 0, 0, 2] - st[items[0], 0, 0, 2]
            if d_ns > 0 and d_clk > 0:
                rates.append(d_clk / d_ns)
        ghz = float(np.median(rates)) if rates else float("nan")
    ns = cyc / ghz
    gaps = []
    for c in range(min(grid, n)):
        items = np.arange(c, n, grid)
        if len(items) >= 2:
            gaps.append((start[items[1:], :] - end[items[:-1], :]).ravel())
    gap_ns = np.concatenate(gaps) / ghz if gaps else np.array([])
    flat = ns.ravel()
    hist, edges = np.histogram(flat, bins=bins)
    pct = {f"p{q}": float(np.percentile(flat, q)) for q in (10, 50, 90, 99)}
    return {"ghz": ghz, "tiles": int(flat.size), "span_ns": pct, "span_mean_ns": float(flat.mean()),
            "gap_ns_median": float(np.median(gap_ns)) if gap_ns.size else None,
            "hist_counts": hist.tolist(), "hist_edges_ns": edges.tolist()}


def store_spans(points, names=("mmdit", "long", "video")):
    """Measured per-tile store-issue spans of the fused kernel against the Burst-Gap and the
    completion-coupled predictions for one wave of tiles (every CTA storing one 128-row tile,
    gap G = the measured median gap between a CTA's bursts)."""
    import torch

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import workloads as W
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = []
    for name in names:
        w = W.WORKLOADS[name]
        g = torch.Generator(device="cuda").manual_seed(0)
        q, k, v = (torch.randn(w.shape(), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        dest = xs.alloc_dest(w.B, w.H, w.S, w.D, w.P, device="cuda")
        xs.attn_a2a_fused(q, k, v, dest)
        spans = xs.attn_a2a_fused_spans(q, k, v, dest)
        torch.cuda.synchronize()
        n_items = spans.shape[0]
        stats = span_stats(spans.cpu().numpy(), min(n_items, sms))
        tile_bytes = 128 * w.D * 2
        gap = stats["gap_ns_median"] if stats["gap_ns_median"] is not None else 0.0
        m = epilogue_models(points, min(n_items, sms), tile_bytes, gap)
        out.append({"workload": name, "S": w.S, "tile_bytes": tile_bytes, "stats": stats,
                    "pred_burst_gap_ns": m["burst_gap_ns"], "pred_completion_coupled_ns": m["completion_coupled_ns"],
                    "pred_T0_ns": m["T0_ns"], "wave_bytes": m["V_bytes"]})
        del q, k, v, dest, spans
    return out


# ----------------------------------------------------------------------------- knee and capacity
def fit_knee(points):
    """Fit T_iss(G) = max(T0_iss, V/R - G) for the points of ONE (K, V), swept over G.

    The drain-dominated side has slope -1 in G by the model; the fit splits the points at
    every candidate knee, takes T0_iss as the mean issue time beyond it and V/R as the mean of
    t + G before it, and keeps the split with the least squared error.  Also fitted, as a
    check of the model rather than a parameter of it: the free slope b of t = a - b G over
    the drain-side points (the model says b = 1).  Returns T0_ns, R_GBps (bytes per ns), the
    knee G* = V/R - T0_iss, the free slope, the number of drain-side points and the RMS
    relative residual of the fitted max(.) curve over all points."""
    pts = sorted(points, key=lambda p: p["G_ns"])
    v = float(pts[0]["V"])
    g = np.array([p["G_ns"] for p in pts], dtype=np.float64)
    t = np.array([p["t_iss_ns"] for p in pts], dtype=np.float64)
    best = None
    for split in range(0, len(pts) + 1):  # points [0, split) drain side, [split, n) floor
        if split == len(pts):
            continue  # no floor point: T0 undetermined
        t0 = float(t[split:].mean())
        a = float((t[:split] + g[:split]).mean()) if split else t0  # a = V / R
        model = np.maximum(t0, a - g)
        sse = float(((model - t) ** 2).sum())
        if best is None or sse < best[0]:
            best = (sse, split, t0, a)
    _, split, t0, a = best
    model = np.maximum(t0, a - g)
    rms = float(np.sqrt(np.mean(((model - t) / t) ** 2)))
    slope = None
    if split >= 2:
        b, _ = np.polyfit(g[:split], t[:split], 1)
        slope = float(-b)
    r = v / a if split else None
    return {"K": pts[0]["K"], "V": int(v), "T0_ns": t0, "R_GBps": r,
            "knee_G_ns": (a - t0) if split else None, "drain_points": int(split),
            "free_slope": slope, "rms_rel_residual": rms}


def fit_capacity(points):
    """Outstanding capacity Q from single bursts with a gap long enough for every earlier
    burst to have drained (points of one K over V, G beyond V/R).  Below Q the burst is
    absorbed at the issue rate I; beyond it issue stalls and the rest goes at the drain rate:
    t(V) = c + V / I for V <= Q, t(V) = c + Q / I + (V - Q) / R_q above.  Q is scanned over
    the measured volumes (and left as "beyond the largest" when one line fits best).
    Returns c, I, R_q, Q and the RMS relative residual."""
    pts = sorted(points, key=lambda p: p["V"])
    v = np.array([p["V"] for p in pts], dtype=np.float64)
    t = np.array([p["t_iss_ns"] for p in pts], dtype=np.float64)
    best = None
    for qi in range(1, len(pts)):  # Q = v[qi]: points 0..qi on the first line
        q = v[qi]
        # least squares in (c, 1/I, 1/R): t = c + min(V, Q)/I + max(V - Q, 0)/R
        a = np.stack([np.ones_like(v), np.minimum(v, q), np.maximum(v - q, 0.0)], axis=1)
        coef, *_ = np.linalg.lstsq(a, t, rcond=None)
        sse = float(((a @ coef - t) ** 2).sum())
        if best is None or sse < best[0] - 1e-12 * sse:
            best = (sse, q, coef)
    _, q, coef = best
    c, inv_i, inv_r = (float(x) for x in coef)
    model = c + np.minimum(v, q) * inv_i + np.maximum(v - q, 0.0) * inv_r
    one = np.polyfit(v, t, 1)
    one_rms = float(np.sqrt(np.mean(((np.polyval(one, v) - t) / t) ** 2)))
    rms = float(np.sqrt(np.mean(((model - t) / t) ** 2)))
    broken = q < v[-1] and inv_r > 0 and inv_i > 0
    return {"c_ns": c, "issue_GBps": 1.0 / inv_i if inv_i > 0 else None,
            "drain_GBps": 1.0 / inv_r if inv_r > 0 else None, "Q_bytes": int(q) if broken else None,
            "rms_rel_residual": rms, "one_line_rms_rel_residual": one_rms,
            "one_line_GBps": 1.0 / one[0] if one[0] > 0 else None}


def knee_sweep(volumes, k: int = 148, r_guess_gbs: float = 7700.0, issue_guess_gbs: float = 8600.0,
               ghz_guess: float = 1.9, n_gaps: int = 17, n_bursts: int = 48, drop: int = 8,
               threads: int = 256, scratch_bytes: int = 2 << 30):
    """T_iss over G densely through [0, 2.5 (V/R - V/I)] for each V at K producers: the knee
    of max(T0_iss, V/R - G) lies at V/R - T0_iss, about V (1/R - 1/I) with I the issue rate
    (R and I guessed from earlier sweeps; the range only has to contain the knee)."""
    import torch

    import ulysses_attention_output_b200 as xs
    scratch = torch.empty(scratch_bytes, dtype=torch.uint8, device="cuda")
    out = []
    for v in volumes:
        vv = (v // (16 * k)) * 16 * k
        g_max_cycles = 2.5 * vv * (1.0 / r_guess_gbs - 1.0 / issue_guess_gbs) * ghz_guess
        for i in range(n_gaps):
            g = int(round(g_max_cycles * i / (n_gaps - 1)))
            out.append(run_point(xs, torch, scratch, k, vv, g, n_bursts, threads, drop))
    del scratch
    return out


def capacity_sweep(volumes, k: int = 148, r_guess_gbs: float = 5000.0, ghz_guess: float = 1.9,
                   n_bursts: int = 12, drop: int = 4, threads: int = 256):
    """Single bursts separated by a gap of 3 V/R (R guessed low): every burst starts drained.
    The scratch ring holds two of the largest bursts (the stores never revisit a line that
    an earlier burst may still hold in L2)."""
    import torch

    import ulysses_attention_output_b200 as xs
    scratch = torch.empty(max(2 << 30, 2 * max(volumes)), dtype=torch.uint8, device="cuda")
    out = []
    for v in volumes:
        vv = (v // (16 * k)) * 16 * k
        g = int(3.0 * vv / r_guess_gbs * ghz_guess)
        out.append(run_point(xs, torch, scratch, k, vv, g, n_bursts, threads, drop))
    del scratch
    return out


def knee_report(points, held_out_v: int):
    """Per-V knee fits of the volumes other than held_out_v, R from their mean, T0_iss(V)
    from a line through their floors, and the prediction of the held-out volume's whole
    T_iss(G) curve against its measurement (relative error per point and RMS)."""
    by_v = {}
    for p in points:
        by_v.setdefault(p["V"], []).append(p)
    fits = {v: fit_knee(pts) for v, pts in sorted(by_v.items())}
    train = [f for v, f in fits.items() if v != held_out_v and f["R_GBps"]]
    r = float(np.mean([f["R_GBps"] for f in train]))
    vols = np.array([f["V"] for f in train], dtype=np.float64)
    floors = np.array([f["T0_ns"] for f in train], dtype=np.float64)
    line = np.polyfit(vols, floors, 1) if len(train) >= 2 else (0.0, floors[0])
    t0_pred = float(np.polyval(line, held_out_v))
    check = []
    for p in sorted(by_v.get(held_out_v, []), key=lambda q: q["G_ns"]):
        pred = predict(t0_pred, r, held_out_v, p["G_ns"])
        check.append({"G_ns": p["G_ns"], "measured_ns": p["t_iss_ns"], "predicted_ns": pred,
                      "rel_err": (pred - p["t_iss_ns"]) / p["t_iss_ns"]})
    rms = float(np.sqrt(np.mean([c["rel_err"] ** 2 for c in check]))) if check else None
    drain_side = [c for c in check if held_out_v / r - c["G_ns"] > t0_pred]
    return {"fits": list(fits.values()), "R_GBps_mean": r,
            "R_GBps_spread": float(np.ptp([f["R_GBps"] for f in train])) if train else None,
            "held_out_V": held_out_v, "T0_pred_ns": t0_pred, "knee_pred_G_ns": held_out_v / r - t0_pred,
            "prediction": check, "prediction_rms_rel": rms,
            "prediction_drain_side_points": len(drain_side)}


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    volumes = [4096 << i for i in range(11)]         # 4 KB .. 4 MB
    producers = [1, 8, 32, 148]
    gaps = [0] + [256 << i for i in range(9)]         # 0, 256 .. 65536 cycles
    if "--large" in argv:                            # bursts beyond the default range
        volumes = [4 << 20, 8 << 20, 16 << 20, 32 << 20, 64 << 20]
        producers = [148]
    threads = 1024 if "--wide" in argv else 256
    if "--knee" in argv:
        # G swept through the knee V/R - T0_iss at 148 producers; 96 MiB is held out of the
        # fit and predicted; then single drained bursts up to 512 MiB for the capacity Q.
        mib = 1 << 20
        kp = knee_sweep([32 * mib, 64 * mib, 96 * mib, 128 * mib], threads=threads)
        held = (96 * mib // (16 * 148)) * 16 * 148
        # A backlog builds at I - R (issue minus drain rate, ~10% of I for local stores), so a
        # capacity Q near the L2 size shows only in bursts of Q / (1 - R/I), over 1 GiB.
        cp = capacity_sweep([v * mib for v in (8, 16, 32, 64, 128, 256, 512, 768, 1024, 1536,
                                               2048, 3072, 4096)], threads=threads, n_bursts=8, drop=2)
        print(json.dumps({"threads_per_producer": threads, "knee_points": kp,
                          "knee": knee_report(kp, held), "capacity_points": cp,
                          "capacity": fit_capacity(cp)}))
        return 0
    pts = sweep(volumes, producers, gaps, threads=threads)
    res = {"threads_per_producer": threads, "points": pts, "fit": fit(pts)}
    if "--fused" in argv:
        res["fused"] = fused_overhead_check(pts)
    if "--spans" in argv:
        res["spans"] = store_spans(pts)
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
