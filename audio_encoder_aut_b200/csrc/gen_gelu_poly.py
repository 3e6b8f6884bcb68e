"""Fits the polynomial behind gelu_fast in aut_ptx.cuh.

GELU(x) = x * Phi(x).  With a = min(|x|, 6):
    Phi(-a) = exp2(-a^2 * log2(e) / 2 + S(a)),
and S(a) = log2(Phi(-a)) + a^2 * log2(e) / 2 is smooth on [0, 6].  S is fitted
by Chebyshev least squares of degree 7 on a dense grid and converted to
monomial coefficients for Horner evaluation in fp32.  Then
    GELU(x) = x * (1 - Phi(-a))  for x >= 0,   x * Phi(-a)  for x < 0,
one exp2 per value.  The script prints the coefficients and the worst
absolute GELU error of an fp32 Horner evaluation against log_ndtr.
Usage: python gen_gelu_poly.py
"""
import numpy as np
from scipy.special import log_ndtr

DEGREE, A_MAX = 7, 6.0


def fit():
    a = np.linspace(0.0, A_MAX, 200001)
    c = np.log2(np.e) / 2
    s = log_ndtr(-a) / np.log(2) + c * a * a
    cheb = np.polynomial.chebyshev.Chebyshev.fit(a, s, DEGREE, domain=[0, A_MAX])
    coef = cheb.convert(kind=np.polynomial.Polynomial, domain=[0, A_MAX], window=[0, A_MAX]).coef
    return a, coef.astype(np.float32)


def worst_error(a, coef):
    af = a.astype(np.float32)
    acc = np.full_like(af, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        acc = (acc * af + coef[k]).astype(np.float32)
    t = (acc - np.float32(np.log2(np.e) / 2) * af * af).astype(np.float32)
    h = np.exp2(t.astype(np.float64))
    href = np.exp(log_ndtr(-a))
    return max(np.abs(a * (h - href)).max(), np.abs(a * ((1 - h) - (1 - href))).max())


if __name__ == "__main__":
    a, coef = fit()
    print("coefficients of a^0 .. a^%d:" % DEGREE)
    print(", ".join("%.9ef" % c for c in coef))
    print("max |GELU error| (fp32 Horner): %.3e" % worst_error(a, coef))
