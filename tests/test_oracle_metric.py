"""Pins of the oracle's error measure, oracle.rel_frobenius(a, b) = ||a - b||_F / ||b||_F.

Every GPU parity assertion goes through this function, so it is pinned on its
own: hand-computed values, the direction of the normalisation (b is the
reference), its zero-reference convention, shape independence, and a
brute-force sum of squares in exact rational arithmetic.  Three plausible
slips (dividing by ||a||, comparing b with itself, returning the numerator
alone) are planted in local copies and must fail at least one pin.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _exact_rel(a, b):
    """sqrt(sum (a-b)^2 / sum b^2) with the sums taken exactly (Fractions)."""
    num = sum((Fraction(float(p)) - Fraction(float(q))) ** 2 for p, q in zip(np.ravel(a), np.ravel(b)))
    den = sum(Fraction(float(q)) ** 2 for q in np.ravel(b))
    return math.sqrt(num / den)


def _pins(fn):
    """Return the list of pin names that `fn` fails (empty when it passes all)."""
    bad = []
    # hand-computed: a - b = (0, 2, 2), ||b|| = 1  ->  sqrt(8)
    if abs(fn(np.array([1.0, 2.0, 2.0]), np.array([1.0, 0.0, 0.0])) - math.sqrt(8.0)) > 1e-15:
        bad.append("hand_value")
    # normalised by the reference b, not by a: (2,0) vs (1,0) is 1; swapped it is 1/2
    if abs(fn(np.array([2.0, 0.0]), np.array([1.0, 0.0])) - 1.0) > 1e-15:
        bad.append("normalised_by_b")
    if abs(fn(np.array([1.0, 0.0]), np.array([2.0, 0.0])) - 0.5) > 1e-15:
        bad.append("normalised_by_b_swapped")
    # equal arrays give exactly zero; a 3-4-5 difference scaled by ||b|| = 10
    if fn(np.full((3, 4), 1.5), np.full((3, 4), 1.5)) != 0.0:
        bad.append("equal_is_zero")
    if abs(fn(np.array([3.0, 4.0]) + np.array([6.0, 8.0]), np.array([6.0, 8.0])) - 0.5) > 1e-15:
        bad.append("pythagorean")
    # zero reference: the measure is the absolute norm of a (documented convention)
    if abs(fn(np.array([3.0, 4.0]), np.zeros(2)) - 5.0) > 1e-15:
        bad.append("zero_reference")
    # shape independence: a 3-D array and its flattening give the same value
    rng = np.random.default_rng(7)
    a = rng.standard_normal((2, 3, 4))
    b = rng.standard_normal((2, 3, 4))
    if fn(a, b) != fn(a.ravel(), b.ravel()):
        bad.append("shape_independent")
    # brute force in exact arithmetic on random data, mixed float32 / float64 inputs
    a32 = rng.standard_normal((5, 7)).astype(np.float32)
    b64 = a32.astype(np.float64) + 1e-3 * rng.standard_normal((5, 7))
    if abs(fn(a32, b64) - _exact_rel(a32, b64)) > 1e-12 * _exact_rel(a32, b64):
        bad.append("exact_bruteforce")
    # a single differing element: |d| / ||b||
    b = np.arange(1.0, 11.0)
    a = b.copy()
    a[4] += 0.25
    if abs(fn(a, b) - 0.25 / math.sqrt(385.0)) > 1e-15:
        bad.append("single_element")
    return bad


def test_rel_frobenius_passes_every_pin():
    assert _pins(oracle.rel_frobenius) == []


def _divides_by_a(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm((a - b).ravel()) / np.linalg.norm(a.ravel()))


def _compares_b_with_b(a, b):
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm((b - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def _numerator_only(a, b):
    return float(np.linalg.norm((np.asarray(a, np.float64) - np.asarray(b, np.float64)).ravel()))


@pytest.mark.parametrize("mutant", [_divides_by_a, _compares_b_with_b, _numerator_only])
def test_planted_mistakes_fail_a_pin(mutant):
    assert _pins(mutant) != []
