"""The tensor-core epilogue evaluates GELU through the erf form of
Abramowitz & Stegun, Handbook of Mathematical Functions, eq. 7.1.28:
erf(x) = 1 - (1 + a1 x + ... + a6 x^6)^-16 for x >= 0, |error| <= 3e-7.
This test reads the six coefficients from the kernel source and checks the
form against math.erf in float64 over the range where GELU is not yet
saturated, so a mistyped coefficient fails here rather than inside the
GPU tolerance."""

import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_coefficients():
    src = open(os.path.join(ROOT, "group_wise_dft_b200", "csrc", "tc_transforms.cuh")).read()
    body = src[src.index("float2 gelu_erf2(float2 v)"):]
    body = body[:body.index("\n}\n")]
    # Horner chain from a6 down to a1, then the constant 1
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    assert len(vals) == 7, vals          # a6 (start) + five fma steps + the constant 1
    a6, a5, a4, a3, a2, a1, one = vals
    assert one == 1.0
    return [a1, a2, a3, a4, a5, a6]


def erf_form(x, a):
    p = 1.0 + sum(c * x ** (k + 1) for k, c in enumerate(a))
    return 1.0 - p ** -16


def test_erf_form_within_published_bound():
    a = kernel_coefficients()
    xs = np.linspace(0.0, 6.0, 60001)
    err = max(abs(erf_form(float(x), a) - math.erf(float(x))) for x in xs)
    assert err <= 3.0e-7, err


def test_gelu_from_form_matches_exact_gelu():
    a = kernel_coefficients()
    for v in np.linspace(-8.0, 8.0, 3201):
        v = float(v)
        r = (1.0 + sum(c * (abs(v) / math.sqrt(2)) ** (k + 1) for k, c in enumerate(a))) ** -16
        h = 0.5 * v * r
        g = v - h if v >= 0 else h
        exact = 0.5 * v * (1.0 + math.erf(v / math.sqrt(2)))
        assert abs(g - exact) <= 3.0e-7 * max(1.0, abs(v)), (v, g, exact)
