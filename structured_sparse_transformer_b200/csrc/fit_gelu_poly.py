"""Derives the polynomial the GEMM epilogues use for the Gaussian tail.

The epilogues evaluate erfc(z) = exp(-z^2) * R(z) with R(z) = erfc(z) exp(z^2)
(the scaled complementary error function, smooth and decreasing from 1).  R is
approximated on z in [0, 4] by a degree-12 Chebyshev least-squares fit,
rewritten as a polynomial in u = z/2 - 1 (|u| <= 1) for Horner evaluation in
fp32.  Run to print the coefficients (low to high) and the fp32 error bound.
"""
import numpy as np
from numpy.polynomial import chebyshev as C
from scipy.special import erfcx

Z_MAX, DEGREE = 4.0, 12


def fit():
    z = np.linspace(0.0, Z_MAX, 200001)
    u = 2.0 * z / Z_MAX - 1.0
    coeffs = C.cheb2poly(C.chebfit(u, erfcx(z), DEGREE))
    c32 = coeffs.astype(np.float32)
    acc = np.full(u.shape, c32[-1], dtype=np.float32)
    u32 = u.astype(np.float32)
    for k in range(DEGREE - 1, -1, -1):
        acc = (acc * u32 + c32[k]).astype(np.float32)
    err = float(np.max(np.abs(acc - erfcx(z)) / erfcx(z)))
    return c32, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients (u^0 .. u^12):", ", ".join(f"{v:.9e}f" for v in c))
    print(f"max relative error of the fp32 Horner evaluation on [0, {Z_MAX}]: {err:.2e}")
