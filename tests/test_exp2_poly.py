"""The FMA-pipe exp2 of the attention softmax (CPU only).

Re-runs the minimax fit of ``csrc/fit_exp2_poly.py``, checks that the float32 literals in
``csrc/attn.cu`` are that fit, and bounds the relative error of the kernel's float32
evaluation order (clamp, 1.5*2^23 shifter rounding, Horner FMAs, exponent add) against
numpy's exp2 over the whole input range the softmax produces, including the clamp region.
The bound (2^-13) sits well below half a bf16 ulp (2^-9), the precision P is stored in.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "ulysses_attention_output_b200", "csrc")


def load_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def kernel_literals():
    text = open(os.path.join(CSRC, "attn.cu")).read()
    m = re.search(r"kC1 = (0x[0-9a-f]+)u, kC2 = (0x[0-9a-f]+)u, kC3 = (0x[0-9a-f]+)u", text)
    assert m, "coefficient literals not found in attn.cu"
    return np.array([1.0] + [np.array([int(h, 16)], dtype=np.uint32).view(np.float32)[0]
                             for h in m.groups()], dtype=np.float32)


def test_literals_are_the_fit():
    fit = load_fit()
    coeffs, err = fit.fit()
    assert err < 1.1e-4
    np.testing.assert_array_equal(coeffs.astype(np.float32), kernel_literals())


def test_float32_evaluation_error_bound():
    fit = load_fit()
    c32 = kernel_literals()
    x = np.concatenate([np.linspace(-126.0, 8.0, 1_000_001), np.arange(-126, 9, dtype=np.float64),
                        np.arange(-126, 8, dtype=np.float64) + 0.5])
    got = fit.eval_f32(c32, x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float32).astype(np.float64)) - 1.0)
    assert rel.max() < 2.0 ** -13
    # integers are exact (p(0) = 1)
    ints = np.arange(-126, 9, dtype=np.float64)
    np.testing.assert_array_equal(fit.eval_f32(c32, ints), np.exp2(ints).astype(np.float32))


def test_clamp_region_and_masked_inputs_give_zero_or_tiny():
    fit = load_fit()
    c32 = kernel_literals()
    got = fit.eval_f32(c32, np.array([-np.inf, -1e30, -500.0, -127.0]))
    np.testing.assert_array_equal(got, np.zeros(4, dtype=np.float32))
    tiny = fit.eval_f32(c32, np.array([-126.9, -126.5, -126.2]))
    assert (tiny >= 0).all() and (tiny < 2.0 ** -125).all()
