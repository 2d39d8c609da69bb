"""Pins of the comparison metric every parity test uses (oracle.parity_errors).

The metric is the one the tolerance is stated in: relative L2 error
||y - y_ref||_2 / ||y_ref||_2 and max |y - y_ref| / max |y_ref|, over the whole
output and, for M > 1, per row (tests/helpers.assert_parity).  Each expected
value below is worked out by hand; planted mistakes in the metric (dividing by
the wrong norm, an unnormalised max error, a squared norm, the wrong zero
branch) are checked to fail these pins.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import qlinear_oracle as qo
from tests.helpers import MAX_ABS_TOL, REL_L2_TOL, assert_parity


def test_three_four_five():
    # y_ref = (3, 4): ||y_ref|| = 5, max |y_ref| = 4; y - y_ref = (0, 1): ||.|| = 1, max = 1
    rel, mabs = oracle.parity_errors(np.array([3.0, 5.0]), np.array([3.0, 4.0]))
    assert rel == 0.2
    assert mabs == 0.25


def test_sign_flip_and_scale():
    # y = -y_ref: ||y - y_ref|| = ||2 y_ref|| = 10, max |.| = 8 -> (2, 2)
    rel, mabs = oracle.parity_errors(np.array([-3.0, -4.0]), np.array([3.0, 4.0]))
    assert (rel, mabs) == (2.0, 2.0)
    # both errors are invariant under a common scale, including negative ones
    r = np.array([[1.0, -2.0, 2.0], [0.5, 0.0, -4.0]])
    y = r + np.array([[0.01, 0.0, -0.02], [0.0, 0.03, 0.0]])
    base = oracle.parity_errors(y, r)
    for c in (1024.0, -0.125):
        got = oracle.parity_errors(c * y, c * r)
        assert got[0] == pytest.approx(base[0], rel=1e-15)
        assert got[1] == pytest.approx(base[1], rel=1e-15)


def test_two_dimensional_output_is_one_vector():
    # [[1, 2], [2, 4]] against [[1, 2], [2, 0]]: ||y_ref|| = 3, ||diff|| = 4, max |y_ref| = 2
    rel, mabs = oracle.parity_errors(np.array([[1.0, 2.0], [2.0, 4.0]]),
                                     np.array([[1.0, 2.0], [2.0, 0.0]]))
    assert rel == pytest.approx(4.0 / 3.0, rel=1e-15)
    assert mabs == 2.0


def test_identical_and_zero_reference():
    assert oracle.parity_errors(np.array([1.5, -2.0]), np.array([1.5, -2.0])) == (0.0, 0.0)
    # y_ref = 0 (x = 0): the relative measures have no denominator; both fall back to the
    # absolute error, so only y = 0 passes the tolerance
    assert oracle.parity_errors(np.zeros(4), np.zeros(4)) == (0.0, 0.0)
    rel, mabs = oracle.parity_errors(np.array([0.0, 3.0, 4.0]), np.zeros(3))
    assert (rel, mabs) == (5.0, 4.0)


def test_fp16_input_is_compared_in_fp64():
    # fp16 y and fp32 reference: 2049 is not an fp16 value (fp16(2049) = 2048)
    y = np.array([2048.0], dtype=np.float16)
    rel, mabs = oracle.parity_errors(y, np.array([2049.0], dtype=np.float32))
    assert rel == pytest.approx(1.0 / 2049.0, rel=1e-15)
    assert mabs == pytest.approx(1.0 / 2049.0, rel=1e-15)


def test_assert_parity_checks_every_row():
    # row 1 is wrong by 50 % but is 1000x smaller than row 0: the whole output passes,
    # the per-row check must not
    r = np.array([[1000.0, -800.0, 600.0], [1.0, 1.0, -1.0]])
    y = r.copy()
    y[1] *= 1.5
    rel, mabs = oracle.parity_errors(y, r)
    assert rel <= REL_L2_TOL and mabs <= MAX_ABS_TOL
    with pytest.raises(AssertionError, match="row 1"):
        assert_parity(y, r)
    assert_parity(y, r, per_row=False)


def test_tolerance_edges():
    # an error of half the relative bound passes; one above both bounds fails
    r = np.array([1.0, 0.0])
    assert_parity(np.array([1.0 + REL_L2_TOL / 2, 0.0]), r, per_row=False)
    with pytest.raises(AssertionError):
        assert_parity(np.array([1.0 + 1.5 * MAX_ABS_TOL, 0.0]), r, per_row=False)


# ---------------------------------------------------------------------------
# planted mistakes in the metric: each must break at least one pin above


def _mut_divide_by_y(y, y_ref):
    y = y.astype(np.float64)
    r = y_ref.astype(np.float64)
    den = np.linalg.norm(y)
    rel = float(np.linalg.norm(y - r) / den) if den > 0 else float(np.linalg.norm(y - r))
    return rel, float(np.abs(y - r).max() / np.abs(r).max())


def _mut_unnormalised_max(y, y_ref):
    y = y.astype(np.float64)
    r = y_ref.astype(np.float64)
    den = np.linalg.norm(r)
    rel = float(np.linalg.norm(y - r) / den) if den > 0 else float(np.linalg.norm(y - r))
    return rel, float(np.abs(y - r).max())


def _mut_squared_norm(y, y_ref):
    y = y.astype(np.float64)
    r = y_ref.astype(np.float64)
    d = float(np.sum((y - r) ** 2))
    den = float(np.sum(r ** 2))
    mref = float(np.abs(r).max())
    return (d / den if den > 0 else d), float(np.abs(y - r).max()) / (mref if mref > 0 else 1.0)


def _mut_zero_ref_passes(y, y_ref):
    y = y.astype(np.float64)
    r = y_ref.astype(np.float64)
    den = np.linalg.norm(r)
    if den == 0:
        return 0.0, 0.0
    return float(np.linalg.norm(y - r) / den), float(np.abs(y - r).max() / np.abs(r).max())


def _mut_fp16_compare(y, y_ref):
    # compares in the precision of y: the reference is rounded to fp16 first
    r = y_ref.astype(y.dtype).astype(np.float64)
    y = y.astype(np.float64)
    den = np.linalg.norm(r)
    mref = float(np.abs(r).max())
    return (float(np.linalg.norm(y - r) / den) if den > 0 else 0.0,
            float(np.abs(y - r).max()) / (mref if mref > 0 else 1.0))


PINS = [test_three_four_five, test_sign_flip_and_scale, test_two_dimensional_output_is_one_vector,
        test_identical_and_zero_reference, test_fp16_input_is_compared_in_fp64]


def _pins_hold():
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            return False
    return True


def test_unmutated_metric_passes_its_pins():
    assert _pins_hold()


@pytest.mark.parametrize("mutant", [_mut_divide_by_y, _mut_unnormalised_max, _mut_squared_norm,
                                    _mut_zero_ref_passes, _mut_fp16_compare])
def test_planted_metric_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(qo, "parity_errors", mutant)
    monkeypatch.setattr(oracle, "parity_errors", mutant)
    assert not _pins_hold(), mutant.__name__


def test_sqrt_of_sum_of_squares_by_hand():
    # an irrational case: y_ref = (1, 1, 1, 1), y = (1, 1, 1, 2): ||diff|| = 1, ||y_ref|| = 2
    rel, _ = oracle.parity_errors(np.array([1.0, 1.0, 1.0, 2.0]), np.ones(4))
    assert rel == 0.5
    rel, _ = oracle.parity_errors(np.array([2.0, 1.0]), np.array([1.0, 1.0]))
    assert rel == pytest.approx(1.0 / math.sqrt(2.0), rel=1e-15)
