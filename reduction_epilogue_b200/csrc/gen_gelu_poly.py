"""Coefficients of the polynomial GELU used by the fused epilogue on a
clamped input range (epilogue (a), whose Hardtanh bounds its GELU input).

GELU(t) = t/2 + t/2 * erf(t / sqrt 2).  The second term is even in t, so on
|t| <= T it is written t^2 * Q(t^2) with Q a polynomial of degree D in
z = t^2; Q is the least-squares fit, weighted to the absolute error of the
GELU, on Chebyshev nodes of [0, T] evaluated in fp64 with math.erf.  The
kernel then evaluates GELU(t) = fma(t^2, Q(t^2), t/2): D + 1 FMAs, no
exponential or division.

    python gen_gelu_poly.py      # prints the table that gelu_poly2() in fle_kernel.cuh holds
"""
import math

import numpy as np

T = 2.0      # the pages' Hardtanh bound: epilogue (a) feeds GELU values in [-2, 2]
D = 7        # degree of Q in z = t^2


def fit(T=T, D=D, m=600):
    t = T * (np.cos(np.pi * (np.arange(m) + 0.5) / m) + 1) / 2
    t = np.concatenate([t, [T]])
    r = np.array([0.5 * v * math.erf(v / math.sqrt(2.0)) for v in t])  # = t^2 Q(t^2)
    A = np.vstack([t ** (2 * k + 2) for k in range(D + 1)]).T
    c, *_ = np.linalg.lstsq(A, r, rcond=None)
    return c


def check(c, T=T):
    t = np.linspace(-T, T, 200001)
    z = t * t
    q = np.zeros_like(t)
    for ck in c[::-1]:
        q = q * z + ck
    approx = z * q + 0.5 * t
    exact = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2.0))) for v in t])
    return float(np.abs(approx - exact).max())


if __name__ == "__main__":
    c = fit()
    print("// Q(z), z = t^2, lowest degree first (gen_gelu_poly.py: T = %g, D = %d; fp64 max |error| %.1e)"
          % (T, D, check(c)))
    print("constexpr float kGeluPolyQ[%d] = {" % (D + 1))
    for ck in c:
        print("    %.9ef," % ck)
    print("};")
