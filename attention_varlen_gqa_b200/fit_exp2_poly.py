"""Fit the cubic used for 2^f, f in [-1/2, 1/2], in the prefill softmax.

Part of the exponentials are computed on the FMA pipe instead of the MUFU
unit: x = n + f with n = round(x) (Cody-Waite split), 2^x = 2^n * p(f).  p is
the degree-3 polynomial minimising the maximum relative error of p(f) / 2^f on
[-1/2, 1/2], found with Lawson's iteratively reweighted least squares on
Chebyshev nodes.  Run this script to reproduce the coefficients written into
csrc/common.cuh (kExp2C0..kExp2C3) and the error bound the tests check.
"""
import numpy as np


def fit(degree=3, nodes=4001, iters=400):
    f = np.cos(np.linspace(0.0, np.pi, nodes)) * 0.5
    t = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / t[:, None]
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        e = A @ c - 1.0
        w = w * np.abs(e)
        w /= w.sum()
    err = np.abs(np.vander(f, degree + 1, increasing=True) @ c / t - 1.0).max()
    return c, err


if __name__ == "__main__":
    c, err = fit()
    c32 = c.astype(np.float32)
    for i, x in enumerate(c32):
        print(f"kExp2C{i} = {float(x)!r}f  // 0x{int(np.float32(x).view(np.uint32)):08x}")
    print(f"max relative error {err:.3e}")
