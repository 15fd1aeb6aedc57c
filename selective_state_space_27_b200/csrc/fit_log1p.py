"""Fit the polynomial behind the kernels' softplus: log1p(e) ~= e * p(e) on [0, 1].

softplus(v) = max(v, 0) + log1p(exp(-|v|)) needs log1p on [0, 1]. The kernels
evaluate it as e * p(e) with p of degree DEG in Horner form, so that the only
transcendental is the ex2 that produced e. The coefficients below come from a
weighted least-squares Chebyshev fit of log1p(e)/e, reweighted towards the
minimax solution (Lawson's iteration), converted to the monomial basis and
rounded to float32. The script prints them and the largest relative error of
log1p measured in float32 Horner evaluation on a fine grid of [0, 1].

    python fit_log1p.py [DEG]     (the kernels use DEG = 6: max rel. error 1.7e-6)
"""
import sys

import numpy as np
from numpy.polynomial import chebyshev as cheb


def fit(deg: int):
    x = (np.cos(np.linspace(0.0, np.pi, 4000)) + 1.0) / 2.0
    f = np.where(x == 0, 1.0, np.log1p(x) / np.where(x == 0, 1.0, x))
    w = np.ones_like(x)
    for _ in range(60):
        c = cheb.chebfit(2 * x - 1, f, deg, w=w)
        err = cheb.chebval(2 * x - 1, c) - f
        w = w * (np.abs(err) / np.abs(err).max()) ** 0.5 + 1e-12
    poly_t = np.polynomial.Polynomial(cheb.cheb2poly(c))
    coef = poly_t(np.polynomial.Polynomial([-1.0, 2.0])).coef       # in e, low to high
    c32 = coef.astype(np.float32)
    e = np.linspace(0.0, 1.0, 400001).astype(np.float32)
    acc = np.full_like(e, c32[-1])
    for ck in c32[-2::-1]:
        acc = (acc * e + ck).astype(np.float32)
    approx = (acc * e).astype(np.float64)
    ref = np.log1p(e.astype(np.float64))
    rel = np.abs(approx - ref) / np.where(ref == 0, 1.0, ref)
    return c32, float(rel.max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 6
    c32, err = fit(deg)
    print(f"degree {deg}: max relative error of log1p {err:.3e}")
    print("coefficients, highest degree first:")
    for ck in c32[::-1]:
        print(f"  {float(ck)!r}f")
