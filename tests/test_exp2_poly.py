"""The FMA-pipe exp2 used for part of the softmax exponentials (forward and,
at d = 64, backward): its coefficients in common.cuh are the ones the
committed fit produces, and the float32 evaluation
(same steps as the kernel) stays within the fit's relative-error bound of
numpy's exp2 over the whole range the kernel uses."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_115_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("__device__ __forceinline__ float2 exp2_pair_fma"):]
    body = body[:body.index("\n}\n")]
    c3, c2 = map(float, re.search(r"ffma2\(pk2\(([-0-9.e]+)f, \1f\), f, pk2\(([-0-9.e]+)f", body).groups())
    c1 = float(re.search(r"ffma2\(pp, f, pk2\(([-0-9.e]+)f", body).group(1))
    return np.array([1.0, c1, c2, c3], dtype=np.float32)


def test_kernel_coefficients_match_fit():
    g = _gen()
    fit = g.fit().astype(np.float32)
    got = _kernel_coefficients()
    assert np.allclose(got, fit, rtol=2e-7, atol=0), (got, fit)


def test_float32_evaluation_error_bound():
    g = _gen()
    coef = _kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32),
                        np.array([-0.5, 0.5, 0.0, -1.0, 7.999], dtype=np.float32)])
    got = g.evaluate_f32(coef, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 1.1e-4
    assert np.all(got > 0)


def test_polynomial_is_exact_at_zero_and_continuous_at_half():
    g = _gen()
    coef = _kernel_coefficients()
    v = g.evaluate_f32(coef, np.array([0.0, 0.4999999, 0.5000001, -3.5, -3.4999998], dtype=np.float32))
    assert v[0] == 1.0
    assert abs(v[1] / v[2] - 1) < 3e-4  # the two sides of a rounding boundary agree
    assert abs(v[3] / v[4] - 1) < 3e-4
