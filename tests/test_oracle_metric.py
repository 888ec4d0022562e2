"""Pins of the parity metric itself, oracle.rel_frobenius (no GPU).

Every parity verdict in this repository goes through this function, so it is
pinned against values worked out by hand: a metric that divided by the wrong
norm, dropped the square root, compared only part of the array or let a NaN
pass would loosen every parity test at once."""
import math

import numpy as np

import oracle


def test_hand_computed_two_by_two():
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    ref = np.array([[1.0, 2.0], [3.0, 5.0]])
    # ||x - ref||_F = 1, ||ref||_F = sqrt(1 + 4 + 9 + 25) = sqrt(39)
    assert oracle.rel_frobenius(x, ref) == 1.0 / math.sqrt(39.0)
    # the denominator is the reference's norm, not the candidate's (sqrt(30))
    assert oracle.rel_frobenius(ref, x) == 1.0 / math.sqrt(30.0)


def test_whole_array_and_square_root():
    # three 2x2 blocks: the metric is over every element at once
    ref = np.arange(1.0, 13.0).reshape(3, 2, 2)
    x = ref.copy()
    x[0, 0, 0] += 3.0
    x[2, 1, 1] -= 4.0
    # sum of squared differences 9 + 16 = 25; sum of squares 1^2 + ... + 12^2 = 650
    assert abs(oracle.rel_frobenius(x, ref) - 5.0 / math.sqrt(650.0)) < 1e-15
    # a difference in the last block alone is still seen
    y = ref.copy()
    y[2, 1, 1] += 1.0
    assert oracle.rel_frobenius(y, ref) > 0.0


def test_scale_invariance_and_sign():
    rng = np.random.default_rng(7)
    ref = rng.standard_normal((5, 7))
    x = ref + 1e-3 * rng.standard_normal((5, 7))
    e = oracle.rel_frobenius(x, ref)
    for c in (1e-6, 0.5, 3.0, 1e6):
        assert abs(oracle.rel_frobenius(c * x, c * ref) - e) <= 1e-12 * e
    assert oracle.rel_frobenius(ref, ref) == 0.0
    assert oracle.rel_frobenius(-ref, ref) == 2.0
    assert oracle.rel_frobenius(np.zeros_like(ref), ref) == 1.0


def test_zero_reference():
    z = np.zeros((3, 3))
    assert oracle.rel_frobenius(z, z) == 0.0
    x = z.copy()
    x[1, 2] = 1e-300
    assert oracle.rel_frobenius(x, z) == math.inf


def test_non_finite_values_fail_every_bound():
    ref = np.ones((4, 4))
    for bad in (math.nan, math.inf, -math.inf):
        x = ref.copy()
        x[2, 3] = bad
        e = oracle.rel_frobenius(x, ref)
        assert not (e <= 1e-4) and not (e <= 2e-2)


def test_float32_inputs_are_measured_in_float64():
    # a float32 candidate against a float64 reference: the error of the
    # float32 rounding itself, not a rounded-away zero
    ref = np.array([1.0 + 2.0 ** -30, 1.0])
    x = ref.astype(np.float32)
    assert oracle.rel_frobenius(x, ref) == 2.0 ** -30 / math.sqrt((1.0 + 2.0 ** -30) ** 2 + 1.0)
