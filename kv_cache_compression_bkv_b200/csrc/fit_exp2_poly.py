"""Fit the cubic used by score_tc.cu to evaluate 2^f on the FMA pipe.

Method: Cody-Waite range reduction x = j + f with j = rint(x) and f in
[-0.5, 0.5], then a polynomial p(f) ~ 2^f.  The coefficients below come from a
Lawson-weighted least-squares fit (iteratively reweighted toward an
equioscillating relative error) on a dense grid, done here from scratch; the
printout reports the maximum relative error of the float32 Horner evaluation.

Run: python fit_exp2_poly.py
"""
import numpy as np


def fit(deg: int, iters: int = 60):
    f = np.linspace(-0.5, 0.5, 40001)
    t = 2.0 ** f
    V = np.vander(f, deg + 1, increasing=True)
    w = 1.0 / t
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * w[:, None], t * w, rcond=None)
        err = (V @ c - t) / t
        w = w * np.sqrt(np.abs(err) + 1e-30)
        w /= w.max()
    c32 = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.full_like(ff, c32[deg])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    return c32, float(np.max(np.abs(p.astype(np.float64) - t) / t))


if __name__ == "__main__":
    for deg in (3, 4):
        c, e = fit(deg)
        print(f"degree {deg}: coefficients {[float(x) for x in c]}  max rel err {e:.3e}")
