"""Fit the cubic that kv_cache_compression_bkv_b200/csrc/score_tc.cu uses to
evaluate 2^f on the FMA pipe (test infrastructure: test_exp2_route.py checks
the kernel's constants against this fit and emulates its route).

Method: Cody-Waite range reduction x = j + f with j = rint(x) and f in
[-0.5, 0.5], then a polynomial p(f) ~ 2^f.  The coefficients below come from a
Lawson-weighted least-squares fit (iteratively reweighted toward an
equioscillating relative error) on a dense grid, done here from scratch; the
printout reports the maximum relative error of the float32 Horner evaluation.

It also emulates, in float32, the whole FMA-pipe route score_tc.cu takes for
2^(v * kz - m): the saturating map of x from [-126, 128] onto [0, 1], the
reduction by the 1.5 * 2^23 constant, the cubic and the exponent insertion
(`exp2_route`), and reports its error over the range the kernel uses.

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


def _rn(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma(a, b, c):
    # fused multiply-add of float32 operands: the exact product and sum in
    # float64 (exact for these magnitudes up to one final rounding), rounded once
    return _rn(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def exp2_route(v, kz, m, coeffs):
    """float32 emulation of 2^(v * kz - m) by the kernel's FMA-pipe route.
    coeffs = (c0, c1, c2, c3) of the cubic, lowest order first."""
    c0, c1, c2, c3 = (np.float32(c) for c in coeffs)
    inv = _rn(1.0 / 254.0)
    base = np.float32(12582912.0 - 126.0)
    a = _rn(np.float32(kz) * inv)
    b = _fma(-np.float32(m), inv, _rn(np.float32(126.0) * inv))
    with np.errstate(all="ignore"):
        y = _fma(_rn(v), a, b)
        y = np.where(np.isnan(y), np.float32(0), np.clip(y, np.float32(0), np.float32(1)))
        y = y.astype(np.float32)
        t = _fma(y, np.float32(254), base)
        u = _fma(t, np.float32(-1), base)
        f = _fma(y, np.float32(254), u)
        p = _fma(_fma(_fma(f, c3, c2), f, c1), f, c0)
    bits = (p.view(np.uint32).astype(np.uint64)
            + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def route_error(coeffs, kz=0.08838835 * 1.4426950408889634, lo=-125.0, hi=64.0, n=400001):
    """Max relative error of exp2_route against 2^x over x in [lo, hi], for a
    few references m."""
    worst = 0.0
    for m in (0.0, 37.5, -12.25, 150.0):
        x = np.linspace(lo, hi, n)
        v = _rn((x + m) / np.float64(np.float32(kz)))
        exact = np.asarray(v, np.float64) * np.float64(np.float32(kz)) - m
        r = exp2_route(v, kz, m, coeffs).astype(np.float64)
        worst = max(worst, float(np.max(np.abs(r / 2.0 ** exact - 1))))
    return worst


if __name__ == "__main__":
    for deg in (3, 4):
        c, e = fit(deg)
        print(f"degree {deg}: coefficients {[float(x) for x in c]}  max rel err {e:.3e}")
    c, _ = fit(3)
    print(f"FMA-pipe route (map, reduction, cubic, exponent): max rel err "
          f"{route_error(c):.3e} over x in [-125, 64]")
