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
