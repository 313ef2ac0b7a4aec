"""Pins for the cyclic oracle (CPU only).

The oracle applies the dense expanded matrix; every check below reaches its
expected value another way: explicit summation of the definition, numpy's FFT
(the convolution theorem), numpy matmul, an impulse response, the shift
invariant and the counts the pages print.
"""

import json
import os

import numpy as np
import pytest

import oracle
from tests import pins

TOL = 1e-12


@pytest.fixture
def rng():
    return np.random.default_rng(12345)


def test_bruteforce_definition(rng):
    assert pins.pin_bruteforce(oracle.cyclic_forward, rng) < TOL


def test_single_channel_is_circular_convolution(rng):
    assert pins.pin_fft_single_channel(oracle.cyclic_forward, rng) < TOL


def test_trivial_group_is_matmul(rng):
    assert pins.pin_n1_matmul(oracle.cyclic_forward, rng) < TOL


def test_convolution_theorem_half_spectrum(rng):
    assert pins.pin_convolution_theorem(oracle.cyclic_forward, rng) < 1e-11


def test_impulse_response_is_weight(rng):
    assert pins.pin_impulse(oracle.cyclic_forward, rng) < TOL


def test_cyclic_shift_equivariance(rng):
    assert pins.pin_shift(oracle.cyclic_forward, rng) < TOL


def test_dense_matrix_is_block_circulant(rng):
    W = rng.standard_normal((3, 2, 8))
    Wd = oracle.cyclic_dense_matrix(W)
    N = 8
    for o in range(3):
        for i in range(2):
            blk = Wd[o * N:(o + 1) * N, i * N:(i + 1) * N]
            for g in range(N):
                # each row is the previous one rotated right by one slot
                assert np.array_equal(blk[g], np.roll(blk[0], g))


def test_counts_match_pages(golden_dir):
    with open(os.path.join(golden_dir, "pages_figures.json")) as f:
        gold = json.load(f)
    c4 = oracle.cyclic_counts(4, 16, 16)
    assert c4["real_gemms"] == gold["p4_real_gemms"]["value"]
    assert c4["dense_gemms"] == gold["p4_dense_gemms"]["value"]
    ratio = c4["dense_gemms"] / c4["real_gemms"]
    assert abs(ratio - gold["p4_theoretical_speedup"]["value"]) < gold["p4_theoretical_speedup"]["tol"]
    assert c4["dense_params"] // c4["params"] == gold["p4_param_ratio"]["value"]
    # exact MAC law for even N: (2N - 2) Cin Cout per token
    for N in (2, 4, 8, 16):
        c = oracle.cyclic_counts(N, 160, 96)
        assert c["fourier_macs"] == (2 * N - 2) * 160 * 96
        assert c["dense_macs"] == N * N * 160 * 96


def test_fp64_exactness_scale():
    """fp64 oracle vs the fp64 FFT route sits far below the pages' fp32 1e-7."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 8, 8))
    W = rng.standard_normal((8, 8, 8)) / 8.0
    X = np.fft.rfft(x, axis=-1)
    Y = np.einsum("oik,tik->tok", np.fft.rfft(W, axis=-1), X)
    ref = np.fft.irfft(Y, n=8, axis=-1)
    assert oracle.rel_frobenius(oracle.cyclic_forward(x, W), ref) < 1e-14
