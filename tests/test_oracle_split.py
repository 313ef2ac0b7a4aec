"""Pins for the negacyclic oracle and the even/odd split of C_2N (CPU only).

The negacyclic layer is the product modulo z^N + 1; for Cin = Cout = 1 it is
checked against numpy polynomial multiplication folded with that sign.  The
split C_2N = (C_N cyclic on x_h + x_{h+N}) and (C_N negacyclic on
x_h - x_{h+N}) is checked against the cyclic oracle, which builds the dense
C_2N matrix directly.
"""

import numpy as np
import pytest

import oracle


def _polymul_mod_zn_plus_1(a, b):
    """(a * b) mod (z^N + 1) for coefficient vectors a, b of length N (index = power)."""
    N = len(a)
    full = np.convolve(a, b)                # powers 0 .. 2N - 2
    out = full[:N].copy()
    out[: len(full) - N] -= full[N:]        # z^(N + j) = -z^j
    return out


@pytest.mark.parametrize("N", [1, 2, 3, 4, 8, 16])
def test_negacyclic_single_channel_is_polynomial_product(N):
    rng = np.random.default_rng(N)
    x = rng.standard_normal((3, 1, N))
    W = rng.standard_normal((1, 1, N))
    y = oracle.negacyclic_forward(x, W)
    for t in range(3):
        ref = _polymul_mod_zn_plus_1(W[0, 0], x[t, 0])
        assert np.max(np.abs(y[t, 0] - ref)) < 1e-12


@pytest.mark.parametrize("N,Cin,Cout", [(1, 3, 2), (2, 2, 3), (4, 3, 5), (8, 4, 6)])
def test_c2n_splits_into_cyclic_and_negacyclic_halves(N, Cin, Cout):
    rng = np.random.default_rng(100 + N)
    x = rng.standard_normal((5, Cin, 2 * N))
    W = rng.standard_normal((Cout, Cin, 2 * N))
    y = oracle.cyclic_forward(x, W)                         # the C_2N layer, dense
    e = x[..., :N] + x[..., N:]
    d = x[..., :N] - x[..., N:]
    ye = oracle.cyclic_forward(e, W[..., :N] + W[..., N:])
    yo = oracle.negacyclic_forward(d, W[..., :N] - W[..., N:])
    assert np.max(np.abs(y[..., :N] - 0.5 * (ye + yo))) < 1e-12
    assert np.max(np.abs(y[..., N:] - 0.5 * (ye - yo))) < 1e-12


def test_split_catches_a_sign_mistake():
    # the same identity with the negacyclic half replaced by a cyclic one fails
    rng = np.random.default_rng(7)
    N = 8
    x = rng.standard_normal((4, 3, 2 * N))
    W = rng.standard_normal((2, 3, 2 * N))
    y = oracle.cyclic_forward(x, W)
    e, d = x[..., :N] + x[..., N:], x[..., :N] - x[..., N:]
    ye = oracle.cyclic_forward(e, W[..., :N] + W[..., N:])
    wrong = oracle.cyclic_forward(d, W[..., :N] - W[..., N:])
    assert np.max(np.abs(y[..., :N] - 0.5 * (ye + wrong))) > 1e-3
