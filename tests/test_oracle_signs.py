"""Pins of the oracle's sign convention for singular pairs (canonical_signs).

An SVD fixes each singular pair (u_i, v_i) only up to a common sign.  The convention: row i
of B (a right singular vector) is negated, with column i of A, when its entry of largest
magnitude is negative.  These checks do not compare with the CUDA path's own helper; they
pin the convention by hand-worked values and by the properties that define it, chosen so
that the plausible slips fail: flipping B's rows without A's columns (A @ B changes),
flipping columns of B instead of rows, or keying on the largest signed entry instead of the
largest magnitude."""
import numpy as np
import pytest

import oracle.starkv_oracle as O


def test_hand_worked_2x3():
    # row 0: largest magnitude is -3 (negative) -> flipped; row 1: largest is 5 -> kept
    A = np.array([[1.0, 2.0],
                  [3.0, 4.0],
                  [5.0, 6.0]])
    B = np.array([[1.0, -3.0, 2.0],
                  [-4.0, 0.5, 5.0]])
    A2, B2 = O.canonical_signs(A, B)
    np.testing.assert_array_equal(B2, [[-1.0, 3.0, -2.0], [-4.0, 0.5, 5.0]])
    np.testing.assert_array_equal(A2, [[-1.0, 2.0], [-3.0, 4.0], [-5.0, 6.0]])


def test_largest_magnitude_not_largest_value():
    # the largest signed entry of the row is 2 (positive), but the largest magnitude is -7:
    # the row must be flipped
    B = np.array([[2.0, -7.0, 1.0]])
    _, B2 = O.canonical_signs(None, B)
    np.testing.assert_array_equal(B2, [[-2.0, 7.0, -1.0]])


def test_rows_not_columns():
    # a column-wise convention would flip column 1 (its largest magnitude, -6, is negative)
    # and leave row 1 alone; the row-wise one flips row 1 only
    B = np.array([[3.0, 1.0],
                  [0.5, -6.0]])
    _, B2 = O.canonical_signs(None, B)
    np.testing.assert_array_equal(B2, [[3.0, 1.0], [-0.5, 6.0]])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_properties_on_random_factors(seed):
    g = np.random.default_rng(seed)
    m, r, n = 9, 5, 7
    A = g.standard_normal((m, r))
    B = g.standard_normal((r, n))
    A2, B2 = O.canonical_signs(A, B)
    # the product is unchanged (A's columns flipped with B's rows)
    np.testing.assert_allclose(A2 @ B2, A @ B, rtol=0, atol=1e-14)
    # each row of B has a positive entry of largest magnitude
    idx = np.argmax(np.abs(B2), axis=1)
    assert np.all(B2[np.arange(r), idx] > 0)
    # every row and column changed by a sign only
    flip = np.sign(B2[:, 0] / B[:, 0])
    np.testing.assert_array_equal(np.abs(flip), 1.0)
    np.testing.assert_array_equal(B2, B * flip[:, None])
    np.testing.assert_array_equal(A2, A * flip[None, :])
    # idempotent: a second application changes nothing
    A3, B3 = O.canonical_signs(A2, B2)
    np.testing.assert_array_equal(A3, A2)
    np.testing.assert_array_equal(B3, B2)
    # the inputs are not modified in place
    A0, B0 = A.copy(), B.copy()
    O.canonical_signs(A, B)
    np.testing.assert_array_equal(A, A0)
    np.testing.assert_array_equal(B, B0)


def test_svd_sign_ambiguity_resolved():
    # two SVDs of one matrix that differ by the signs of their singular pairs give the same
    # factors after the convention
    g = np.random.default_rng(7)
    W = g.standard_normal((6, 4))
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    signs = np.array([1.0, -1.0, -1.0, 1.0])
    A1, B1 = O.canonical_signs(U * s, Vt)
    A2, B2 = O.canonical_signs(U * s * signs, Vt * signs[:, None])
    np.testing.assert_allclose(A1, A2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(B1, B2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(A1 @ B1, W, rtol=0, atol=1e-12)
