"""Coefficients of the polynomial part of the attention kernel's software exp2.

Method: Cody-Waite style range reduction 2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2],
and 2^f approximated by a polynomial fitted by weighted least squares on Chebyshev nodes of
[-1/2, 1/2] (a near-minimax fit of the relative error), evaluated with Horner's rule. The
constant term is pinned to 1 so that 2^0 is exact. Run this file to print the coefficients
that exp2_poly2() in the attention kernel (csrc/attn_sm100.cuh) uses and the fit's maximum relative error.
"""
import numpy as np

DEGREE = 3


def fit(degree=DEGREE, nodes=4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    # p(f) = 1 + sum_{i>=1} c_i f^i; minimise sum ((p - 2^f) / 2^f)^2
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    coeffs = np.concatenate([[1.0], c])
    grid = np.linspace(-0.5, 0.5, 200001)
    approx = np.polyval(coeffs[::-1], grid)
    err = np.max(np.abs(approx / np.exp2(grid) - 1.0))
    return coeffs, err


if __name__ == "__main__":
    for deg in (2, 3, 4, 5):
        c, e = fit(deg)
        print(deg, " ".join(f"{np.float32(x).item()!r}f" for x in c), f"max rel err {e:.3e}")
