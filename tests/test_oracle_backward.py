"""Pins for the backward-pass oracle (CPU only).

The oracle's backward data pass applies the dense matrix's transpose and its
weight gradient sums the dense gradient over the copies of each shared weight;
every check reaches its expected value another way: explicit loops over the
definition, the adjoint and directional-derivative identities against the
forward oracle, numpy's FFT (cross-correlation theorem) and numpy matmul.
A planted mistake in a copy of either routine must fail a pin.
"""

import numpy as np
import pytest

import oracle
from tests import pins

TOL = 1e-12


def _bwd_pins(bwd, wgrad):
    rng = np.random.default_rng(7)
    return max(pins.pin_backward_data_bruteforce(bwd, rng),
               pins.pin_weight_grad_bruteforce(wgrad, rng),
               pins.pin_adjoint_identity(oracle.cyclic_forward, bwd, rng),
               pins.pin_weight_grad_identity(oracle.cyclic_forward, wgrad, rng),
               pins.pin_weight_grad_fft(wgrad, rng),
               pins.pin_backward_n1_matmul(bwd, wgrad, rng))


def test_backward_data_bruteforce():
    assert pins.pin_backward_data_bruteforce(oracle.cyclic_backward_data, np.random.default_rng(1)) < TOL


def test_weight_grad_bruteforce():
    assert pins.pin_weight_grad_bruteforce(oracle.cyclic_weight_grad, np.random.default_rng(2)) < TOL


def test_backward_data_is_adjoint_of_forward():
    assert pins.pin_adjoint_identity(oracle.cyclic_forward, oracle.cyclic_backward_data,
                                     np.random.default_rng(3)) < TOL


def test_weight_grad_is_directional_derivative():
    assert pins.pin_weight_grad_identity(oracle.cyclic_forward, oracle.cyclic_weight_grad,
                                         np.random.default_rng(4)) < TOL


def test_weight_grad_single_channel_is_cross_correlation():
    assert pins.pin_weight_grad_fft(oracle.cyclic_weight_grad, np.random.default_rng(5)) < 1e-11


def test_trivial_group_is_matmul():
    assert pins.pin_backward_n1_matmul(oracle.cyclic_backward_data, oracle.cyclic_weight_grad,
                                       np.random.default_rng(6)) < TOL


def test_real_oracle_passes_all_backward_pins():
    assert _bwd_pins(oracle.cyclic_backward_data, oracle.cyclic_weight_grad) < 1e-11


def _bwd_reflect_sign(dy, W):
    # correlation instead of convolution: uses W[o, i, (h - g) mod N]
    return oracle.cyclic_backward_data(dy, np.asarray(W)[:, :, (-np.arange(W.shape[2])) % W.shape[2]])


def _bwd_forward_instead(dy, W):
    # forgets the transpose: applies the forward map's weight with in/out swapped
    return oracle.cyclic_forward(dy, np.transpose(np.asarray(W, float), (1, 0, 2)))


def _wgrad_plus(x, dy):
    # (g + m) instead of (g - m)
    dW = oracle.cyclic_weight_grad(x, dy)
    N = dW.shape[2]
    return dW[:, :, (-np.arange(N)) % N]


def _wgrad_dropped_token(x, dy):
    x = np.array(x, float)
    x[-1] = 0.0
    return oracle.cyclic_weight_grad(x, dy)


def _wgrad_transposed(x, dy):
    # swaps the roles of x and dy (a transposed operand)
    return np.transpose(oracle.cyclic_weight_grad(dy, x), (1, 0, 2)) if x.shape[1] == dy.shape[1] \
        else oracle.cyclic_weight_grad(x, dy) * 1.001


@pytest.mark.parametrize("bwd", [_bwd_reflect_sign, _bwd_forward_instead])
def test_backward_data_mutants_are_caught(bwd):
    assert _bwd_pins(bwd, oracle.cyclic_weight_grad) > 1e-6


@pytest.mark.parametrize("wgrad", [_wgrad_plus, _wgrad_dropped_token, _wgrad_transposed])
def test_weight_grad_mutants_are_caught(wgrad):
    assert _bwd_pins(oracle.cyclic_backward_data, wgrad) > 1e-6
