"""Pins for the parity metric itself (no GPU).

Every forward parity assertion goes through ``oracle.rel_max_err``: the largest
absolute error over the whole output divided by the root mean square of the
reference output (the tolerance metric of the hot-path statement: "max abs
error relative to output RMS").  These cases are worked by hand, so a metric
that took the mean instead of the max, the max (or the mean of absolute values)
instead of the RMS as the denominator, or dropped the square root, fails here.
"""
import math

import numpy as np
import pytest

import oracle as O


def test_hand_worked_pair():
    # |got - ref| = [0, 2] -> max 2; RMS(ref) = sqrt((1 + 0) / 2) = sqrt(0.5)
    assert O.rel_max_err([1.0, 2.0], [1.0, 0.0]) == pytest.approx(2.0 / math.sqrt(0.5), rel=1e-15)


def test_max_not_mean_and_rms_not_max():
    ref = np.array([3.0, 4.0])
    got = ref + np.array([0.1, -0.5])
    # max |err| = 0.5 (the mean would be 0.3); RMS(ref) = sqrt(12.5) = 3.5355...
    # (max |ref| = 4 and mean |ref| = 3.5 give other values; so does RMS^2 = 12.5)
    want = 0.5 / math.sqrt(12.5)
    got_err = O.rel_max_err(got, ref)
    assert got_err == pytest.approx(want, rel=1e-14)
    for wrong in (0.3 / math.sqrt(12.5), 0.5 / 4.0, 0.5 / 3.5, 0.5 / 12.5):
        assert abs(got_err - wrong) > 1e-3 * want


def test_whole_tensor_not_per_row():
    # rows with very different scales: the denominator is the RMS of every element together
    ref = np.array([[10.0, 0.0], [0.0, 0.0]])
    got = ref.copy()
    got[1, 1] = 1.0
    # RMS = sqrt(100 / 4) = 5, max |err| = 1
    assert O.rel_max_err(got, ref) == pytest.approx(0.2, rel=1e-15)


def test_symmetric_sign_and_exact_match():
    ref = np.array([1.0, -2.0, 2.0])
    assert O.rel_max_err(ref, ref) == 0.0
    up = O.rel_max_err(ref + np.array([0.0, 0.25, 0.0]), ref)
    down = O.rel_max_err(ref - np.array([0.0, 0.25, 0.0]), ref)
    assert up == down == pytest.approx(0.25 / math.sqrt(3.0), rel=1e-15)


def test_empty_arrays():
    assert O.rel_max_err(np.zeros((0, 4)), np.zeros((0, 4))) == 0.0


def test_zero_rms_reference():
    z = np.zeros(5)
    assert O.rel_max_err(z, z) == 0.0
    # any error against an all-zero reference is far beyond every tolerance
    assert O.rel_max_err(z + 1e-12, z) > 1e6


def test_non_finite_output_never_passes():
    ref = np.array([1.0, 2.0])
    for bad in (np.nan, np.inf):
        err = O.rel_max_err(np.array([1.0, bad]), ref)
        assert not (err <= 2e-2)
