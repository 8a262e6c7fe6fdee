"""Pins of the pass criterion every fp16/bf16 parity result goes through.

The stated bounds are a maximum absolute error of 1e-3*sqrt(K) and a maximum
relative error of 1e-2.  These cases sit just inside and just outside each
bound on its own, so swapped tolerances, a summed (allclose) form, a bound
taken on the wrong operand or a comparison that lets NaN through fails one
of them.
"""
import math

import numpy as np
import pytest

from oracle import compare


def test_atol_is_one_thousandth_of_sqrt_k():
    assert compare.atol_for(256) == pytest.approx(0.016, abs=0, rel=1e-15)
    assert compare.atol_for(4096) == pytest.approx(0.064, abs=0, rel=1e-15)
    assert compare.atol_for(10 ** 6) == pytest.approx(1.0, abs=0, rel=1e-15)
    assert compare.RTOL == 1e-2


def test_absolute_bound_just_inside_and_outside():
    K = 256                                   # atol = 0.016
    ref = np.zeros((3, 4))
    inside = ref + 0.0159
    outside = ref.copy()
    outside[1, 2] = 0.0161
    assert compare.check_close(inside, ref, K)["ok"]
    rep = compare.check_close(outside, ref, K)
    assert not rep["ok"] and rep["n_bad"] == 1 and rep["first_bad"] == (1, 2)
    # also below the reference: the error is an absolute value
    assert not compare.check_close(ref - 0.0161, ref, K)["ok"]


def test_absolute_bound_holds_for_large_references_too():
    # |ref| = 100 with an error of 0.5: within 1 % but 30x the absolute bound;
    # the summed form atol + rtol*|ref| would accept it
    K = 256
    ref = np.full(8, 100.0)
    assert not compare.check_close(ref + 0.5, ref, K)["ok"]
    assert compare.check_close(ref + 0.015, ref, K)["ok"]


def test_relative_bound_just_inside_and_outside():
    K = 10 ** 6                               # atol = 1.0: the relative bound decides
    ref = np.array([1.5, -2.0, 3.0])
    ok = ref * (1 + 0.0099 * np.sign(ref))
    bad = ok.copy()
    bad[1] = -2.0 * 1.0101
    assert compare.check_close(ok, ref, K)["ok"]
    rep = compare.check_close(bad, ref, K)
    assert not rep["ok"] and rep["n_bad_rel"] == 1 and rep["n_bad_abs"] == 0
    assert rep["max_rel"] == pytest.approx(0.0101, rel=1e-9)


def test_relative_bound_is_waived_at_or_below_atol():
    K = 10 ** 6                               # atol = 1.0
    ref = np.array([0.5, -1.0, 0.0])          # |ref| <= atol: only the absolute bound applies
    got = ref + np.array([0.9, 0.99, -0.999])
    assert compare.check_close(got, ref, K)["ok"]
    # one ulp above atol the relative bound applies again
    ref2 = np.array([math.nextafter(1.0, 2.0)])
    assert not compare.check_close(ref2 + 0.5, ref2, K)["ok"]


def test_relative_error_is_taken_against_the_reference():
    # y below ref: 0.999 % of ref passes, though it is 1.009 % of y;
    # y above ref: 1.005 % of ref fails, though it is 0.995 % of y
    K = 10 ** 6
    assert compare.check_close(np.array([1.6 * (1 - 0.00999)]), np.array([1.6]), K)["ok"]
    assert not compare.check_close(np.array([1.5 * 1.01005]), np.array([1.5]), K)["ok"]


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_non_finite_fails(bad):
    ref = np.ones(5)
    got = ref.copy()
    got[3] = bad
    rep = compare.check_close(got, ref, 256)
    assert not rep["ok"] and rep["n_nonfinite"] == 1 and rep["first_bad"] == (3,)
    # a non-finite reference fails as well
    assert not compare.check_close(ref, got, 256)["ok"]


def test_shape_mismatch_raises():
    with pytest.raises(ValueError):
        compare.check_close(np.zeros((4, 3)), np.zeros((3, 4)), 64)
    with pytest.raises(ValueError):
        compare.check_close(np.zeros(12), np.zeros((3, 4)), 64)


def test_exact_match_reports_zero_errors():
    ref = np.linspace(-3, 3, 50).reshape(5, 10)
    rep = compare.check_close(ref.copy(), ref, 768)
    assert rep["ok"] and rep["max_abs"] == 0.0 and rep["max_rel"] == 0.0 and rep["first_bad"] is None
