"""The FMA-pipe exp2 of the attention kernel (sm100.cuh: ex2_poly), emulated in fp32 on the CPU.

Same operation sequence as the device code: clamp at -125, round-to-integer by
adding 1.5*2^23, degree-3 polynomial in Horner form with fused multiply-adds,
exponent-field add. Checked against exp2 in fp64: relative error below 1e-4
(the fit's bound is 7.5e-5; fp32 rounding adds a few ulp) over the whole input
range the kernel uses, exact powers of two at integers.
"""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "context_long_sequence_cp_b200", "csrc", "sm100.cuh")


def coefficients():
    body = open(SRC).read().split("ex2_poly(float x)")[1].split("}")[0]
    return [np.float32(float(c)) for c in re.findall(r"([0-9.]+e[-+][0-9]+)f", body)]


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def ex2_poly(x):
    c3, c2, c1, c0 = coefficients()
    x = np.maximum(np.float32(x), np.float32(-125.0))
    t = np.float32(x + np.float32(12582912.0))
    f = np.float32(x - np.float32(t - np.float32(12582912.0)))
    p = fma32(fma32(fma32(c3, f, c2), f, c1), f, c0)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return np.uint32(bits).view(np.float32)


def test_poly_relative_error_over_kernel_range():
    xs = np.concatenate([np.linspace(-125.0, 8.0, 200001, dtype=np.float32),
                         np.random.default_rng(0).uniform(-30, 8, 100000).astype(np.float32)])
    got = np.array([ex2_poly(x) for x in xs[::37]], dtype=np.float64)
    ref = np.exp2(xs[::37].astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1e-4, rel.max()


def test_poly_at_integers_and_halves():
    for n in range(-120, 9):
        assert abs(float(ex2_poly(np.float32(n))) / 2.0 ** n - 1) < 1e-4
        assert abs(float(ex2_poly(np.float32(n + 0.5))) / 2.0 ** (n + 0.5) - 1) < 1e-4


def test_poly_coefficients_match_generator():
    import importlib.util
    spec = importlib.util.spec_from_file_location("gen", os.path.join(os.path.dirname(SRC), "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.remez(3)
    assert err < 8e-5
    assert np.allclose(np.array(coefficients()[::-1], dtype=np.float64), c.astype(np.float64), rtol=1e-6)
