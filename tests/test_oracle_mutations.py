"""The pins must catch plausible mistakes.  Each test plants one mistake in a
local copy of an oracle routine (on the CPU, never in the product) and checks
that at least one pin rejects the copy while the real oracle passes."""

import math

import numpy as np
import pytest

import oracle
from tests import pins


def _cyclic_pins(fwd):
    rng = np.random.default_rng(99)
    return max(pins.pin_bruteforce(fwd, rng), pins.pin_fft_single_channel(fwd, rng),
               pins.pin_convolution_theorem(fwd, rng), pins.pin_impulse(fwd, rng),
               pins.pin_shift(fwd, rng), pins.pin_n1_matmul(fwd, rng))


def _dense_fwd(make_m):
    def fwd(x, W):
        x = np.asarray(x, float)
        W = np.asarray(W, float)
        T, Cin, N = x.shape
        Cout = W.shape[0]
        g = np.arange(N)[:, None]
        h = np.arange(N)[None, :]
        blocks = make_m(W, g, h, N)
        Wd = blocks.transpose(0, 2, 1, 3).reshape(Cout * N, Cin * N)
        return (x.reshape(T, -1) @ Wd.T).reshape(T, Cout, N)
    return fwd


def test_real_oracle_passes_all_cyclic_pins():
    assert _cyclic_pins(oracle.cyclic_forward) < 1e-11


@pytest.mark.parametrize("name,make_m", [
    ("correlation_sign", lambda W, g, h, N: W[:, :, (h - g) % N]),
    ("no_wraparound", lambda W, g, h, N: np.where((g - h) >= 0, 1.0, 0.0) * W[:, :, np.clip(g - h, 0, N - 1)]),
    ("off_by_one", lambda W, g, h, N: W[:, :, (g - h + 1) % N]),
    ("slot_transposed", lambda W, g, h, N: W[:, :, (g - h) % N].transpose(0, 1, 3, 2) * 1.0
     if N > 2 else W[:, :, (g - h) % N] * 1.01),
])
def test_cyclic_mutants_are_caught(name, make_m):
    assert _cyclic_pins(_dense_fwd(make_m)) > 1e-6, name


def test_cyclic_dropped_term_is_caught():
    def fwd(x, W):
        y = oracle.cyclic_forward(x, W)
        x2 = np.array(x, float)
        x2[:, -1, :] = 0.0          # drops the last input field's contribution
        return oracle.cyclic_forward(x2, W) if x2.shape[1] > 1 else y * 0.5
    assert _cyclic_pins(fwd) > 1e-6


# ------------------------------------------------------------------ D8 mutants

def _d8_pins(fwd):
    rng = np.random.default_rng(5)
    E = oracle.d8_elements()
    return max(pins.pin_d8_equivariance(fwd, rng, E, oracle.d8_regular_perm),
               pins.pin_d8_closed_forms(fwd, rng, E, oracle.d8_slot, oracle.d8_inv, oracle.d8_mul))


def _d8_variant(share_over="a", back="QT", swap=None, e_index="2i+b"):
    Q = oracle.d8_Q()

    def fwd(x, wA1, wA2, wB1, wB2, wE):
        x = np.asarray(x, float)
        T, F, _ = x.shape
        z = np.einsum("cg,tig->tic", Q, x)
        zo = np.zeros_like(z)
        blocks = [wA1, wA2, wB1, wB2]
        if swap:
            i, j = swap
            blocks[i], blocks[j] = blocks[j], blocks[i]
        for c, w in enumerate(blocks):
            zo[:, :, c] = z[:, :, c] @ np.asarray(w, float).T
        wE = np.asarray(wE, float)
        for p in range(2):
            v = np.empty((T, 2 * F))
            for q in range(2):
                a, b = (p, q) if share_over == "a" else (q, p)
                if e_index == "2i+b":
                    v[:, q::2] = z[:, :, 4 + 2 * a + b]
                else:
                    v[:, q * F:(q + 1) * F] = z[:, :, 4 + 2 * a + b]
            vo = v @ wE.T
            for q in range(2):
                a, b = (p, q) if share_over == "a" else (q, p)
                zo[:, :, 4 + 2 * a + b] = vo[:, q::2] if e_index == "2i+b" else vo[:, q * F:(q + 1) * F]
        if back == "QT":
            return np.einsum("cg,tic->tig", Q, zo)
        return np.einsum("gc,tic->tig", Q, zo)
    return fwd


def test_real_d8_oracle_passes():
    assert _d8_pins(oracle.d8_forward) < 1e-12
    assert _d8_pins(_d8_variant()) < 1e-12


@pytest.mark.parametrize("kw", [
    {"share_over": "b"},          # E block shared over the wrong index
    {"back": "Q"},                # back-transform with Q instead of Q^T
    {"swap": (1, 2)},             # A2 and B1 blocks exchanged
    {"swap": (0, 3)},
])
def test_d8_mutants_are_caught(kw):
    assert _d8_pins(_d8_variant(**kw)) > 1e-6, kw


def test_tanh_gelu_is_caught():
    v = np.linspace(-4, 4, 81)
    tanh_gelu = 0.5 * v * (1 + np.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3)))
    assert np.max(np.abs(tanh_gelu - pins.gelu_reference(v))) > 1e-5
    assert np.max(np.abs(oracle.gelu_exact(v) - pins.gelu_reference(v))) < 1e-15
