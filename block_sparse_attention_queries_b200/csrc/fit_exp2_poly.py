"""Derivation of the cubic used by exp2_poly2() in ab_ptx.cuh.

2^y = 2^n * 2^f with n = round(y) and f = y - n in [-1/2, 1/2] (Cody-Waite
style split); 2^f is approximated by a cubic fitted here for minimal
relative error on [-1/2, 1/2] (weighted least squares on Chebyshev nodes,
reweighted towards equal ripple).  Max relative error 7.5e-5, far below the
2^-9 rounding of the bf16 probabilities the kernel stores.  Run to print the
coefficients (highest degree first)."""
import numpy as np


def fit(deg=3, iters=60):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    w = 1.0 / y
    c = np.polyfit(f, y, deg, w=w)
    for _ in range(iters):
        err = (np.polyval(c, f) - y) / y
        w = w * (np.abs(err) + 1e-18) ** 0.5
        w = w / w.max()
        c = np.polyfit(f, y, deg, w=w / y)
    ff = np.linspace(-0.5, 0.5, 200001)
    return c, float(np.abs(np.polyval(c, ff) / np.exp2(ff) - 1).max())


if __name__ == "__main__":
    c, e = fit()
    print([float(np.float32(x)) for x in c], "max rel err", e)
