"""The GPU parity checks' own logic (CPU only): the format-limited split of the O check must
still catch real errors."""

import numpy as np
import pytest

from parity import TOL_O_MAX, assert_fwd_ok, bf16_ulp, fwd_errors


def _err(o_ref, delta):
    o_ref = np.asarray(o_ref, np.float64)
    return fwd_errors(o_ref + np.asarray(delta), np.zeros(1), o_ref, np.zeros(1))


def test_bf16_ulp():
    assert np.allclose(bf16_ulp(np.array([1.0, 1.9, 2.0, 4.0, 7.9, 0.25])),
                       [2 ** -7, 2 ** -7, 2 ** -6, 2 ** -5, 2 ** -5, 2 ** -9])


def test_in_range_error_is_caught():
    ref = np.zeros(1000)
    ref[0] = 3.9
    d = np.zeros(1000)
    d[0] = 1.1 * TOL_O_MAX  # |O| < 4: the plain 1e-2 bound applies
    with pytest.raises(AssertionError):
        assert_fwd_ok(_err(ref, d), "in-range")


def test_format_limited_within_one_ulp_passes_and_beyond_fails():
    ref = np.zeros(1000)
    ref[0] = 5.3
    d = np.zeros(1000)
    d[0] = 0.9 * 2 ** -5  # 0.028 > 1e-2 but within one bf16 ulp at 5.3
    e = _err(ref, d)
    assert e["o_max"] > TOL_O_MAX and e["format_limited"] == 1
    assert_fwd_ok(e, "format-limited")
    d[0] = 1.5 * 2 ** -5
    with pytest.raises(AssertionError):
        assert_fwd_ok(_err(ref, d), "beyond one ulp")


def test_mean_and_lse_bounds():
    ref = np.zeros(100)
    with pytest.raises(AssertionError):
        assert_fwd_ok(_err(ref, np.full(100, 2e-3)), "mean")
    e = fwd_errors(ref, np.array([2e-3]), ref, np.zeros(1))
    with pytest.raises(AssertionError):
        assert_fwd_ok(e, "lse")
