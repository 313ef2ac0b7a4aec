"""CPU pin of the p4 (N = 4) adds-only transforms.

p4_forward and p4_inverse are host-and-device inline functions; this test
compiles a small host program against the library's internal header (nvcc,
no GPU needed), runs them on seeded inputs and compares with numpy's FFT:
to fp32 rounding for random inputs and exactly for small integers, where
every sum is exact.  The forward must give [Re X0, Re X1, Im X1, Re X2] with
X_k = sum_h x_h exp(-2 pi i h k / 4); the inverse must give
y_g = Y0 + (-1)^g Y2 + 2 Re(Y1 exp(2 pi i g / 4)), the one-sided inverse
without the 1/4 (which lives in the weight spectrum).
"""

import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")

HARNESS = r"""
#include <cstdio>
#include "eqlin_internal.cuh"
int main() {
  float v[4], o[4];
  while (scanf("%f %f %f %f", &v[0], &v[1], &v[2], &v[3]) == 4) {
    eqlin::p4_forward(v, o);
    printf("%.9g %.9g %.9g %.9g ", o[0], o[1], o[2], o[3]);
    eqlin::p4_inverse(v, o);
    printf("%.9g %.9g %.9g %.9g\n", o[0], o[1], o[2], o[3]);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("p4")
    src = d / "p4.cu"
    src.write_text(HARNESS)
    exe = d / "p4"
    subprocess.run([nvcc, "-std=c++17", "-I", CSRC, "-I", INCLUDE, "-o", str(exe), str(src)], check=True,
                   capture_output=True)
    return str(exe)


def run(exe, rows):
    inp = "\n".join(" ".join(repr(float(v)) for v in r) for r in rows) + "\n"
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout
    a = np.array([[float(t) for t in line.split()] for line in out.strip().splitlines()])
    return a[:, :4], a[:, 4:]


def reference(rows):
    X = np.fft.fft(rows, axis=-1)
    fwd = np.stack([X[:, 0].real, X[:, 1].real, X[:, 1].imag, X[:, 2].real], axis=-1)
    Y = rows[:, 0] + 0j, rows[:, 1] + 1j * rows[:, 2], rows[:, 3] + 0j
    g = np.arange(4)
    inv = (Y[0][:, None].real + ((-1.0) ** g)[None, :] * Y[2][:, None].real
           + 2 * (Y[1][:, None] * np.exp(2j * np.pi * g / 4)[None, :]).real)
    return fwd, inv


def test_p4_transforms_match_the_dft_on_random_inputs(harness):
    rows = np.random.default_rng(0).standard_normal((200, 4)).astype(np.float32).astype(np.float64)
    fwd, inv = run(harness, rows)
    rf, ri = reference(rows)
    assert np.max(np.abs(fwd - rf)) <= 4e-6 * np.max(np.abs(rf))
    assert np.max(np.abs(inv - ri)) <= 4e-6 * np.max(np.abs(ri))


def test_p4_transforms_are_exact_on_integers(harness):
    rows = np.random.default_rng(1).integers(-1000, 1001, (200, 4)).astype(np.float64)
    fwd, inv = run(harness, rows)
    rf, ri = reference(rows)
    assert np.array_equal(fwd, np.round(rf)) and np.array_equal(inv, np.round(ri))
