"""The FMA-pipe exp of the row statistics (score_tc.cu, exp2_poly2), emulated
in float32 with the coefficients read from the kernel source: its error bound,
and the properties the row statistics' lagged reference relies on -- below
the range the result is a tiny non-negative number (also for -inf and NaN),
above 64 (or with a reference of -inf) it exceeds 2^64, so the block's sum
shows the overflow."""
import importlib.util
import pathlib
import re

import numpy as np
import pytest

CSRC = pathlib.Path(__file__).resolve().parents[1] / "kv_cache_compression_bkv_b200" / "csrc"
HERE = pathlib.Path(__file__).resolve().parent
KZ = np.float32(0.08838835 * 1.4426950408889634)  # (1/sqrt(128)) * log2(e)


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", HERE / "fit_exp2_poly.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coeffs():
    src = (CSRC / "score_tc.cu").read_text()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"(\d\.\d{5,})f", body)]
    assert len(vals) == 8, vals
    c3, c2, c1, c0 = vals[0], vals[2], vals[4], vals[6]
    assert vals == [c3, c3, c2, c2, c1, c1, c0, c0]
    return c0, c1, c2, c3


@pytest.fixture(scope="module")
def fit():
    return _fit_module()


def test_kernel_coefficients_are_the_fit(fit):
    c, err = fit.fit(3)
    assert np.allclose(_kernel_coeffs(), c, rtol=0, atol=2e-8)
    assert err < 8e-5


def test_route_error_bound(fit):
    assert fit.route_error(_kernel_coeffs()) < 1e-4


def test_below_the_range(fit):
    c = _kernel_coeffs()
    x = -np.logspace(np.log10(126.0), 30, 2001)
    for m in (0.0, 40.0):
        v = (x + m) / np.float64(KZ)
        r = fit.exp2_route(v.astype(np.float32), KZ, m, c)
        assert np.all(np.isfinite(r)) and np.all(r >= 0) and np.all(r <= 2.0 ** -125)
    special = np.array([-np.inf, np.nan], dtype=np.float32)
    for m in (0.0, 40.0, -np.inf):
        r = fit.exp2_route(special, KZ, m, c)
        assert np.all(np.isfinite(r)) and np.all(r >= 0) and np.all(r <= 2.0 ** -125)


def test_above_the_range_shows_in_the_sum(fit):
    c = _kernel_coeffs()
    x = np.concatenate([np.linspace(64.5, 300.0, 4001), np.logspace(2.5, 30, 200)])
    for m in (0.0, 40.0):
        v = ((x + m) / np.float64(KZ)).astype(np.float32)
        r = fit.exp2_route(v, KZ, m, c).astype(np.float64)
        assert np.all(r > 2.0 ** 64)
    # the first block of a row: reference -inf, any finite logit
    v = np.linspace(-1e6, 1e6, 1001).astype(np.float32)
    r = fit.exp2_route(v, KZ, -np.inf, c).astype(np.float64)
    assert np.all(r > 2.0 ** 64)


def test_saturated_top_is_just_under_float_max(fit):
    """At the top of the mapped range (x >= 128, or a reference of -inf) the
    saturating map gives y = 1, f = 0 and an exponent of 2^128 inserted into
    p(0): about 2^128, finite and just below FLT_MAX -- so two such terms in a
    sum overflow to inf, which the row statistics treat like any sum above
    2^64 (the block is summed again against a new reference)."""
    c = _kernel_coeffs()
    for m in (0.0, 40.0, -np.inf):
        v = np.array([1e30, 3e4, (200.0 + (0 if np.isinf(m) else m)) / KZ], dtype=np.float32)
        r = fit.exp2_route(v, KZ, m, c)
        assert np.all(np.isfinite(r)), r
        rr = r.astype(np.float64)
        assert np.all(rr > 2.0 ** 127.99) and np.all(rr <= np.finfo(np.float32).max)
        assert np.isinf(np.float32(r[0]) + np.float32(r[1]))
