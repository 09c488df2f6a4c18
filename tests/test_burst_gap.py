"""Burst-Gap model evaluation and fit (CPU only): the fit must recover the parameters of
synthetic sweeps generated from the model itself (T_iss = max(T0_iss(K, V), V/R - G), the
explainer's "Methodik" section), and stamps must convert to nanoseconds correctly."""
import numpy as np

from ulysses_attention_output_b200 import burst_gap as bg


def synthetic(r_gbs=717.0, issue_gbs=3000.0, t_fixed=400.0, noise=0.0, seed=0):
    rng = np.random.default_rng(seed)
    pts = []
    for k in (1, 8, 148):
        for v in [4096 << i for i in range(11)]:
            t0 = t_fixed + v / issue_gbs          # backpressure-free issue cost
            for g in [0.0] + [100.0 * 2 ** i for i in range(10)]:
                t = bg.predict(t0, r_gbs, v, g) * (1 + noise * rng.standard_normal())
                pts.append({"K": k, "V": v, "G_ns": g, "t_iss_ns": t})
    return pts


def test_predict_regimes():
    assert bg.predict(100.0, 1000.0, 1e6, 0.0) == 1000.0            # drain-dominated: V/R
    assert bg.predict(100.0, 1000.0, 1e6, 950.0) == 100.0           # gap covers the drain
    assert bg.predict(100.0, 1000.0, 1e6, 500.0) == 500.0           # partly covered
    assert bg.completion_coupled(1000.0, 1e6) == 1000.0


def test_fit_recovers_parameters():
    r, b, a = 717.0, 3000.0, 400.0
    f = bg.fit(synthetic(r, b, a))
    assert abs(f["R_GBps"] - r) / r < 1e-6
    assert abs(f["T0_ns"]["K=148,V=4096"] - (a + 4096 / b)) < 1e-6
    # knee: largest swept V with V/R <= 1.25 * (a + V/b)
    vols = [4096 << i for i in range(11)]
    expect = max(v for v in vols if v / r <= 1.25 * (a + v / b))
    assert f["Q_bytes"] == expect


def test_fit_tolerates_noise():
    f = bg.fit(synthetic(noise=0.02, seed=3))
    assert abs(f["R_GBps"] - 717.0) / 717.0 < 0.05


def test_issue_times_from_stamps():
    # two producers, 12 bursts; 2 GHz clock; each burst: 500 cycles of issue, 4000 of gap
    k, n, ghz = 2, 12, 2.0
    st = np.zeros((k, n, 4), dtype=np.int64)
    for p in range(k):
        t = 1000 * p
        for i in range(n):
            st[p, i] = [t, t + 500, t + 4500, int((t + 123) / ghz)]
            t += 4600
    issue, gap, clk = bg.issue_times_ns(st, drop=2)
    assert abs(clk - ghz) < 1e-3
    np.testing.assert_allclose(issue, 250.0, rtol=1e-3)
    np.testing.assert_allclose(gap, 2000.0, rtol=1e-3)


def test_epilogue_models():
    pts = synthetic(r_gbs=700.0, issue_gbs=3000.0, t_fixed=400.0)
    m = bg.epilogue_models(pts, 148, 65536, gap_ns=1e5)
    v = 148 * 65536
    assert m["V_bytes"] == v
    # backpressure-free time interpolated in V; gap covers the drain -> Burst-Gap gives T0
    assert abs(m["T0_ns"] - (400.0 + v / 3000.0)) < 1e-6 * m["T0_ns"]
    assert m["burst_gap_ns"] == m["T0_ns"]
    assert abs(m["completion_coupled_ns"] - max(m["T0_ns"], v / 700.0)) < 1e-6 * v
    # no gap: the drain term wins
    z = bg.epilogue_models(pts, 148, 65536, gap_ns=0.0)["burst_gap_ns"]
    assert abs(z - max(m["T0_ns"], v / 700.0)) < 1e-9 * z


def test_span_stats_from_synthetic_stamps():
    # 2 CTAs, 3 items each (items striped: i on CTA i % 2); SM clock 2 GHz.
    ghz, grid, n = 2.0, 2, 6
    st = np.zeros((n, 2, 4, 3), dtype=np.int64)
    item_cycles = 100_000
    for i in range(n):
        c, k = i % grid, i // grid
        for t in range(2):
            for w in range(4):
                t0 = 1_000 + k * item_cycles + 50 * w + 5_000 * t   # warps start staggered
                st[i, t, w, 0] = t0
                st[i, t, w, 1] = t0 + 2_000 + 100 * w               # last warp ends latest
                st[i, t, w, 2] = int(t0 / ghz) + 10_000_000 * c
    r = bg.span_stats(st, grid)
    assert abs(r["ghz"] - ghz) < 1e-3
    # span = max end - min start = (150 + 2000 + 300) - 0 = 2450 cycles = 1225 ns for every tile
    assert r["tiles"] == 12
    assert abs(r["span_ns"]["p50"] - 1225.0) < 1e-6 and abs(r["span_ns"]["p99"] - 1225.0) < 1e-6
    # gap: next item's first start - this item's last end = 100000 - 2450 cycles
    assert abs(r["gap_ns_median"] - (item_cycles - 2450) / ghz) < 1e-6
    assert sum(r["hist_counts"]) == 12
    # an explicit clock rate overrides the estimate
    assert abs(bg.span_stats(st, grid, ghz=1.0)["span_ns"]["p50"] - 2450.0) < 1e-6


# ----------------------------------------------------------------------------- knee and capacity
def knee_points(v, t0, r, gaps, noise=0.0, seed=0, slope=1.0):
    """Points of one (K, V) over G from the model (slope != 1 plants a model violation)."""
    rng = np.random.default_rng(seed)
    out = []
    for g in gaps:
        t = max(t0, v / r - slope * g) * (1 + noise * rng.standard_normal())
        out.append({"K": 148, "V": v, "G_ns": float(g), "t_iss_ns": t})
    return out


def test_fit_knee_recovers_t0_r_and_knee():
    v, t0, r = 64 << 20, 7600.0, 7700.0                  # bytes, ns, bytes/ns (= GB/s)
    gaps = np.linspace(0.0, 2 * v / r, 17)
    f = bg.fit_knee(knee_points(v, t0, r, gaps))
    assert abs(f["R_GBps"] - r) / r < 1e-6
    assert abs(f["T0_ns"] - t0) < 1e-6
    assert abs(f["knee_G_ns"] - (v / r - t0)) < 1e-3
    assert abs(f["free_slope"] - 1.0) < 1e-6
    assert f["rms_rel_residual"] < 1e-9


def test_fit_knee_with_noise_and_a_planted_slope():
    v, t0, r = 128 << 20, 15000.0, 7000.0
    gaps = np.linspace(0.0, 2 * v / r, 33)
    f = bg.fit_knee(knee_points(v, t0, r, gaps, noise=0.01, seed=4))
    assert abs(f["R_GBps"] - r) / r < 0.03
    assert abs(f["free_slope"] - 1.0) < 0.15
    # a drain side of slope 0.5 instead of 1 is not the model: the free slope shows it
    g = bg.fit_knee(knee_points(v, t0, r, gaps, slope=0.5))
    assert abs(g["free_slope"] - 0.5) < 0.05


def test_fit_knee_without_a_drain_regime():
    """Every gap beyond the knee (backpressure-free only): no drain-side points, no R."""
    v, t0 = 8 << 20, 1000.0
    f = bg.fit_knee(knee_points(v, t0, 1e9, np.linspace(0.0, 5000.0, 9)))
    assert f["drain_points"] == 0 and f["R_GBps"] is None and abs(f["T0_ns"] - t0) < 1e-9


def test_knee_report_predicts_a_held_out_volume():
    r, c, issue = 7500.0, 200.0, 8800.0
    mib = 1 << 20
    pts = []
    for v in (32 * mib, 64 * mib, 96 * mib, 128 * mib):
        pts += knee_points(v, c + v / issue, r, np.linspace(0.0, 2 * v / r, 17))
    rep = bg.knee_report(pts, 96 * mib)
    assert abs(rep["R_GBps_mean"] - r) / r < 1e-6
    assert rep["prediction_rms_rel"] < 1e-9
    assert rep["prediction_drain_side_points"] > 0
    # a held-out curve that breaks the model is predicted badly
    bad = [p if p["V"] != 96 * mib else {**p, "t_iss_ns": 1.3 * p["t_iss_ns"]} for p in pts]
    assert bg.knee_report(bad, 96 * mib)["prediction_rms_rel"] > 0.2


def capacity_points(vols, c, issue, q, drain):
    return [{"K": 148, "V": v, "G_ns": 1e6, "t_iss_ns": c + min(v, q) / issue + max(v - q, 0) / drain}
            for v in vols]


def test_fit_capacity_recovers_q():
    mib = 1 << 20
    vols = [v * mib for v in (8, 16, 32, 48, 64, 96, 128, 192, 256, 384, 512)]
    f = bg.fit_capacity(capacity_points(vols, 250.0, 8800.0, 96 * mib, 6000.0))
    assert f["Q_bytes"] == 96 * mib
    assert abs(f["issue_GBps"] - 8800.0) / 8800.0 < 1e-6
    assert abs(f["drain_GBps"] - 6000.0) / 6000.0 < 1e-6
    assert f["rms_rel_residual"] < 1e-9 < f["one_line_rms_rel_residual"]


def test_fit_capacity_without_a_break():
    """One rate over every volume: Q is beyond the largest burst measured."""
    mib = 1 << 20
    vols = [v * mib for v in (8, 16, 32, 64, 128, 256)]
    f = bg.fit_capacity(capacity_points(vols, 250.0, 8000.0, 1 << 40, 8000.0))
    assert f["Q_bytes"] is None or abs(f["issue_GBps"] - f["drain_GBps"]) / 8000.0 < 1e-6
    assert abs(f["one_line_GBps"] - 8000.0) / 8000.0 < 1e-6
