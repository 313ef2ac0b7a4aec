"""Pins for the D8 oracle (CPU only): group axioms, orthogonality of the
change of basis, block diagonalisation of the regular representation, the
equivariance the page requires, group-convolution structure, full rank of the
Fourier parametrisation, closed forms from the character table, exact GELU and
the counts printed on the Quick ViTs page."""

import json
import math
import os

import numpy as np
import pytest

import oracle
from tests import pins

E = oracle.d8_elements()


@pytest.fixture
def rng():
    return np.random.default_rng(2024)


def test_group_axioms():
    r, s, e = (1, 0), (0, 1), (0, 0)
    mul = oracle.d8_mul
    assert mul(mul(mul(r, r), r), r) == e
    assert mul(s, s) == e
    assert mul(mul(s, r), s) == oracle.d8_inv(r)
    for a in E:
        for b in E:
            for c in E:
                assert mul(mul(a, b), c) == mul(a, mul(b, c))
    # the 8 slots are 8 distinct elements
    assert len(set(E)) == 8


def test_irreps_are_homomorphisms():
    for a in E:
        for b in E:
            ab = oracle.d8_mul(a, b)
            assert np.allclose(oracle.d8_rho_E(ab), oracle.d8_rho_E(a) @ oracle.d8_rho_E(b))
            assert np.allclose(oracle.d8_chars_1d(ab), oracle.d8_chars_1d(a) * oracle.d8_chars_1d(b))


def test_characters_match_textbook_table():
    for u in E:
        cls = pins.d8_class(u)
        ch = oracle.d8_chars_1d(u)
        for k, name in enumerate(("A1", "A2", "B1", "B2")):
            assert ch[k] == pins.D8_CHAR_TABLE[name][cls]
        assert np.trace(oracle.d8_rho_E(u)) == pins.D8_CHAR_TABLE["E"][cls]


def test_regular_action_is_a_representation():
    for a in E:
        for b in E:
            Pab = oracle.d8_regular_perm(oracle.d8_mul(a, b))
            assert np.array_equal(Pab, oracle.d8_regular_perm(a) @ oracle.d8_regular_perm(b))


def test_Q_orthogonal():
    Q = oracle.d8_Q()
    assert np.allclose(Q @ Q.T, np.eye(8), atol=1e-15)


def test_Q_block_diagonalises_regular_rep():
    Q = oracle.d8_Q()
    for u in E:
        B = Q @ oracle.d8_regular_perm(u) @ Q.T
        ref = np.zeros((8, 8))
        ref[0:4, 0:4] = np.diag(oracle.d8_chars_1d(u))
        ref[4:8, 4:8] = np.kron(oracle.d8_rho_E(u), np.eye(2))   # rows a act, columns b ride along
        assert np.allclose(B, ref, atol=1e-14)


def test_layer_is_equivariant(rng):
    err = pins.pin_d8_equivariance(oracle.d8_forward, rng, E, oracle.d8_regular_perm)
    assert err < 1e-12


def test_gelu_layer_is_equivariant(rng):
    f = lambda x, *w: oracle.d8_forward(x, *w, fuse_gelu=True)
    assert pins.pin_d8_equivariance(f, rng, E, oracle.d8_regular_perm) < 1e-12


def test_operator_is_group_convolution(rng):
    F = 2
    ws = [rng.standard_normal((F, F)) for _ in range(4)] + [rng.standard_normal((2 * F, 2 * F))]
    K = oracle.d8_dense_operator(*ws).reshape(F, 8, F, 8)
    slot = oracle.d8_slot
    for o in range(F):
        for i in range(F):
            kern = {}
            for g in E:
                for h in E:
                    key = oracle.d8_mul(oracle.d8_inv(g), h)
                    v = K[o, slot(g), i, slot(h)]
                    if key in kern:
                        assert abs(kern[key] - v) < 1e-13
                    kern[key] = v


def test_fourier_parametrisation_has_full_rank():
    """C = 16: the 4*(C/8)^2 + (C/4)^2 = C^2/8 = 32 parameters map onto a
    32-dimensional space of operators, the dimension of all equivariant maps
    on 2 copies of the regular representation (8 * 2^2)."""
    F = 2
    shapes = [(F, F)] * 4 + [(2 * F, 2 * F)]
    nparam = sum(a * b for a, b in shapes)
    assert nparam == (8 * F) ** 2 // 8
    ops = []
    for p in range(nparam):
        flat = np.zeros(nparam)
        flat[p] = 1.0
        ws, off = [], 0
        for a, b in shapes:
            ws.append(flat[off:off + a * b].reshape(a, b))
            off += a * b
        ops.append(oracle.d8_dense_operator(*ws).ravel())
    assert np.linalg.matrix_rank(np.array(ops), tol=1e-9) == nparam == 8 * F * F


def test_closed_forms_from_character_table(rng):
    err = pins.pin_d8_closed_forms(oracle.d8_forward, rng, E, oracle.d8_slot, oracle.d8_inv, oracle.d8_mul)
    assert err < 1e-13


def test_gelu_exact():
    v = np.linspace(-6.0, 6.0, 241)
    assert np.max(np.abs(oracle.gelu_exact(v) - pins.gelu_reference(v))) < 1e-15
    # GELU(1) = Phi(1) = 0.8413447460685429 (standard normal table)
    assert abs(oracle.gelu_exact(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    # odd-part identity GELU(v) - GELU(-v) = v
    assert np.max(np.abs(oracle.gelu_exact(v) - oracle.gelu_exact(-v) - v)) < 1e-14
    assert oracle.gelu_exact(np.array([0.0]))[0] == 0.0


def test_counts_match_pages(golden_dir):
    with open(os.path.join(golden_dir, "pages_figures.json")) as f:
        gold = json.load(f)
    for C in (16, 1280, 8192):
        c = oracle.d8_counts(C)
        assert c["param_ratio"] == gold["d8_param_ratio"]["value"]
        assert abs(c["mult_ratio"] - gold["d8_mult_ratio"]["value"]) < gold["d8_mult_ratio"]["tol"]
        assert c["mults"] == 3 * C * C // 16
