"""Seeded input generators (CPU only): determinism and the stated structure."""
import torch

from ulysses_attention_output_b200 import workloads as W


def test_deterministic_and_bf16():
    a = W.make_qkv(1, 2, 64, 16, seed=5)
    b = W.make_qkv(1, 2, 64, 16, seed=5)
    c = W.make_qkv(1, 2, 64, 16, seed=6)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])


def test_qknorm_rows_have_unit_rms_times_gain():
    q, k, v = W.make_qkv(1, 3, 256, 32, seed=1, structure="qknorm")
    rms = q.float().pow(2).mean(-1).sqrt()
    # gains ~ N(1, 0.1): the RMS of a normalised row times the gain stays near 1
    assert 0.8 < rms.mean().item() < 1.2
    assert rms.std().item() < 0.2
    # V is untouched iid N(0,1)
    assert abs(v.float().std().item() - 1.0) < 0.05


def test_outlier_keys():
    S = 1000
    q, k, _ = W.make_qkv(1, 2, S, 16, seed=2, structure="outliers")
    _, k_plain, _ = W.make_qkv(1, 2, S, 16, seed=2, structure="iid")
    for h in range(2):
        scaled = (k[0, h].float() != k_plain[0, h].float()).any(-1)
        assert int(scaled.sum()) <= S // 100
        rows = scaled.nonzero().flatten()
        torch.testing.assert_close(k[0, h, rows].float(), 8 * k_plain[0, h, rows].float(), rtol=0, atol=0)


def test_workload_table():
    assert [W.WORKLOADS[n].S for n in W.ORDER] == [256, 1024, 4608, 16384, 32768]
    for n in W.ORDER:
        w = W.WORKLOADS[n]
        assert w.S % w.P == 0 and w.H % w.P == 0
    assert W.WORKLOADS["mmdit"].flops == 4 * 24 * 4608 ** 2 * 128


def test_sampled_rows_include_boundaries():
    w = W.WORKLOADS["long"]
    rows = W.sample_rows(w)
    assert rows.shape == (1, 24, 256)
    Sl = w.S // w.P
    for h in range(24):
        r = set(rows[0, h].tolist())
        assert len(r) == 256
        assert {0, w.S - 1} <= r
        for b in range(1, w.P):
            assert {b * Sl - 1, b * Sl} <= r
