"""Coefficients of the polynomial that evaluates 2^f on the FMA pipe.

The forward softmax computes p = 2^x for every score.  The special-function
unit (MUFU ex2) does 16 of those per clock per SM, as many cycles per tile as
the tensor core's own work, so part of the exponentials are evaluated on the
FMA pipe instead, by range reduction plus a polynomial:

    x = n + f,  n = round(x),  f in [-1/2, 1/2]
    2^x = 2^n * p(f),          p(f) ~= 2^f

2^n is applied by adding n to the exponent field of p(f).  p is the degree-3
polynomial with p(0) = 1 that minimises the maximum RELATIVE error on
[-1/2, 1/2]: a weighted least-squares fit on Chebyshev nodes, refined by
Lawson's iteratively reweighted least squares toward the minimax solution.
Run this file to print the coefficients and the error bound that the CUDA
code (fwd.cu, exp2_poly) and tests/test_exp2_poly.py use.
"""
import numpy as np

DEGREE = 3


def fit(degree=DEGREE, iters=200):
    # Chebyshev nodes on [-1/2, 1/2]
    k = np.arange(4000)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))
    target = np.exp2(f)
    # p(f) = 1 + sum_{i>=1} c_i f^i ; fit the c_i
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1)
    b = target - 1.0
    w = np.ones_like(f)
    for _ in range(iters):
        # relative error weighting 1/2^f, Lawson reweighting toward minimax
        sw = np.sqrt(w) / target
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs((1.0 + A @ c) - target) / target
        w = w * (err + 1e-300)
        w = w / w.sum()
    return np.concatenate([[1.0], c])


def evaluate_f32(coef, x):
    """Reference evaluation in float32 with the same steps as the kernel."""
    x = np.asarray(x, dtype=np.float32)
    magic = np.float32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = [np.float32(v) for v in coef]
    p = c[3]
    p = (p * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    coef = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(coef[::-1], f) - np.exp2(f)) / np.exp2(f)
    print("coefficients c0..c3 (float32):")
    for c in coef:
        print(f"  {np.float32(c)!r}  ({c:.17g})")
    print(f"max relative error on [-1/2, 1/2] (exact arithmetic): {rel.max():.3e}")
    xs = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = evaluate_f32(coef.astype(np.float32), xs)
    rel32 = np.abs(got.astype(np.float64) - np.exp2(xs.astype(np.float64))) / np.exp2(xs.astype(np.float64))
    print(f"max relative error, float32 evaluation on [-125, 8]: {rel32.max():.3e}")
