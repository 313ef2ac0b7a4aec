"""Pins for the Fourier-resident D8 MLP oracle (CPU only).

d8_fourier_linear is checked against the regular-domain D8 oracle (square
blocks directly, rectangular ones by zero padding to a square layer); every
function is checked for equivariance under all 8 group elements acting on the
Fourier coordinates as Q P_u Q^T; the GELU round trip is checked against
math.erf applied in the regular domain; the whole block against the
regular-domain composition.  Planted mistakes fail.
"""

import math

import numpy as np
import pytest

import oracle

E = oracle.d8_elements()
Q = oracle.d8_Q()


def _blocks(rng, F_out, F_in, scale=0.3):
    return tuple(rng.standard_normal((F_out, F_in)) * scale for _ in range(4)) + \
        (rng.standard_normal((2 * F_out, 2 * F_in)) * scale,)


def _to_fourier(x):
    return np.einsum("cg,tig->tic", Q, x)


def _to_regular(z):
    return np.einsum("cg,tic->tig", Q, z)


def _pad(blocks, F):
    """Rectangular blocks in the top-left corner of F x F (2F x 2F for E) zero blocks."""
    out = []
    for k, w in enumerate(blocks):
        n = 2 * F if k == 4 else F
        p = np.zeros((n, n))
        p[: w.shape[0], : w.shape[1]] = w
        out.append(p)
    return out


def _regular_linear(x, blocks, F_out):
    """The rectangular layer through the square regular-domain oracle: zero-pad the
    input fields and the blocks, run d8_forward, keep the first F_out fields."""
    T, F_in, _ = x.shape
    F = max(F_in, F_out)
    xp = np.zeros((T, F, 8))
    xp[:, :F_in] = x
    return oracle.d8_forward(xp, *_pad(blocks, F), fuse_gelu=False)[:, :F_out]


def _gelu_erf(v):
    return 0.5 * v * (1.0 + np.vectorize(math.erf)(v / math.sqrt(2.0)))


def _rho(u):
    P = oracle.d8_regular_perm(u)
    return Q @ P @ Q.T


def _equivariance_error(f, z):
    err = 0.0
    for u in E:
        R = _rho(u)
        a = f(np.einsum("dc,tic->tid", R, z))
        b = np.einsum("dc,tic->tid", R, f(z))
        err = max(err, float(np.max(np.abs(a - b))))
    return err


def test_square_fourier_linear_is_the_regular_layer():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 6, 8))
    w = _blocks(rng, 6, 6)
    got = _to_regular(oracle.d8_fourier_linear(_to_fourier(x), *w))
    assert np.max(np.abs(got - oracle.d8_forward(x, *w))) < 1e-12


@pytest.mark.parametrize("F_in,F_out", [(3, 12), (12, 3), (5, 7)])
def test_rectangular_fourier_linear_is_the_padded_regular_layer(F_in, F_out):
    rng = np.random.default_rng(F_in * 31 + F_out)
    x = rng.standard_normal((4, F_in, 8))
    w = _blocks(rng, F_out, F_in)
    got = _to_regular(oracle.d8_fourier_linear(_to_fourier(x), *w))
    assert np.max(np.abs(got - _regular_linear(x, w, F_out))) < 1e-12


def test_fourier_linear_is_equivariant():
    rng = np.random.default_rng(2)
    w = _blocks(rng, 5, 3)
    z = rng.standard_normal((3, 3, 8))
    assert _equivariance_error(lambda v: oracle.d8_fourier_linear(v, *w), z) < 1e-12


def test_gelu_roundtrip_is_gelu_in_the_regular_domain():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 5, 8)) * 2
    got = oracle.d8_gelu_roundtrip(_to_fourier(x))
    assert np.max(np.abs(got - _to_fourier(_gelu_erf(x)))) < 1e-12
    assert _equivariance_error(oracle.d8_gelu_roundtrip, _to_fourier(x)) < 1e-12


def test_mlp_block_is_the_regular_domain_mlp():
    rng = np.random.default_rng(4)
    F, H = 3, 12                                   # C -> 4C -> C
    x = rng.standard_normal((4, F, 8))
    w1, w2 = _blocks(rng, H, F), _blocks(rng, F, H)
    got = _to_regular(oracle.d8_mlp_block(_to_fourier(x), w1, w2))
    ref = _regular_linear(_gelu_erf(_regular_linear(x, w1, H)), w2, F)
    assert np.max(np.abs(got - ref)) < 1e-12
    assert _equivariance_error(lambda v: oracle.d8_mlp_block(v, w1, w2), _to_fourier(x)) < 1e-11


def test_mistakes_are_caught():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 3, 8)) * 2
    z = _to_fourier(x)
    # the round trip taken in the wrong direction (Q^T on the way back)
    wrong_rt = lambda v: np.einsum("cg,tig->tic", Q.T, _gelu_erf(np.einsum("cg,tic->tig", Q.T, v)))
    assert np.max(np.abs(wrong_rt(z) - _to_fourier(_gelu_erf(x)))) > 1e-3
    # E's second row coordinate with a transposed block (not shared)
    w = _blocks(rng, 3, 3)

    def unshared(v):
        out = oracle.d8_fourier_linear(v, *w)
        alt = oracle.d8_fourier_linear(v, *w[:4], w[4].T)
        out[:, :, 6:8] = alt[:, :, 6:8]
        return out
    assert _equivariance_error(unshared, z) > 1e-3
