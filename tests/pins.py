"""Independent checks ("pins") for the fp64 oracle.

Each pin computes its expected value by a route that shares no arithmetic with
the oracle: a direct summation of the definition, a numpy FFT, a numpy matmul,
a closed form, a group-theoretic invariant or a textbook value.  Every pin is a
function of the callable it checks, so the mutation tests can run the same pins
against copies of the oracle with a planted mistake and see them fail.
"""

from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------- cyclic pins


def brute_force_cyclic(x, W):
    """y[t,o,g] = sum_i sum_h W[o,i,(g-h) mod N] x[t,i,h], by explicit loops."""
    T, Cin, N = x.shape
    Cout = W.shape[0]
    y = np.zeros((T, Cout, N))
    for t in range(T):
        for o in range(Cout):
            for g in range(N):
                s = 0.0
                for i in range(Cin):
                    for h in range(N):
                        s += float(W[o, i, (g - h) % N]) * float(x[t, i, h])
                y[t, o, g] = s
    return y


def pin_bruteforce(forward, rng, shapes=((3, 2, 3, 1), (2, 3, 2, 2), (2, 2, 3, 3),
                                          (2, 3, 2, 4), (1, 2, 2, 5), (2, 2, 2, 8))):
    err = 0.0
    for T, Cin, Cout, N in shapes:
        x = rng.standard_normal((T, Cin, N))
        W = rng.standard_normal((Cout, Cin, N))
        err = max(err, np.max(np.abs(forward(x, W) - brute_force_cyclic(x, W))))
    return err


def pin_fft_single_channel(forward, rng, Ns=(2, 3, 4, 7, 8, 16)):
    """Cin = Cout = 1: the layer is textbook circular convolution."""
    err = 0.0
    for N in Ns:
        x = rng.standard_normal((4, 1, N))
        W = rng.standard_normal((1, 1, N))
        ref = np.real(np.fft.ifft(np.fft.fft(W[0, 0])[None, :] * np.fft.fft(x[:, 0, :], axis=-1), axis=-1))
        err = max(err, np.max(np.abs(forward(x, W)[:, 0, :] - ref)))
    return err


def pin_n1_matmul(forward, rng):
    """N = 1: the layer is a plain matrix product y = x W^T."""
    x = rng.standard_normal((5, 4, 1))
    W = rng.standard_normal((3, 4, 1))
    return float(np.max(np.abs(forward(x, W)[:, :, 0] - x[:, :, 0] @ W[:, :, 0].T)))


def pin_convolution_theorem(forward, rng, cases=((4, 3, 5, 4), (3, 4, 2, 8), (2, 3, 3, 16), (2, 2, 3, 5))):
    """Half-spectrum route with numpy's rfft/irfft: per kept bin k,
    Y_k = What_k X_k, then the inverse real transform."""
    err = 0.0
    for T, Cin, Cout, N in cases:
        x = rng.standard_normal((T, Cin, N))
        W = rng.standard_normal((Cout, Cin, N))
        X = np.fft.rfft(x, axis=-1)          # [T, Cin, N//2+1]
        Wh = np.fft.rfft(W, axis=-1)         # [Cout, Cin, N//2+1]
        Y = np.einsum("oik,tik->tok", Wh, X)
        ref = np.fft.irfft(Y, n=N, axis=-1)
        err = max(err, np.max(np.abs(forward(x, W) - ref)))
    return err


def pin_impulse(forward, rng):
    """x = delta at (field i0, slot 0) gives y[o, g] = W[o, i0, g]."""
    Cin, Cout, N = 3, 4, 8
    W = rng.standard_normal((Cout, Cin, N))
    err = 0.0
    for i0 in range(Cin):
        x = np.zeros((1, Cin, N))
        x[0, i0, 0] = 1.0
        err = max(err, np.max(np.abs(forward(x, W)[0] - W[:, i0, :])))
    return err


def pin_shift(forward, rng):
    """Rolling x by s along the group axis rolls y by s (equivariance)."""
    err = 0.0
    for N in (4, 8, 5):
        x = rng.standard_normal((3, 2, N))
        W = rng.standard_normal((3, 2, N))
        y = forward(x, W)
        for s in range(N):
            err = max(err, np.max(np.abs(forward(np.roll(x, s, axis=-1), W) - np.roll(y, s, axis=-1))))
    return err


# ---------------------------------------------------------------- D8 pins
#
# The character table of the order-8 dihedral group, from any group-theory
# text: classes {e}, {r^2}, {r, r^3}, {s, r^2 s}, {r s, r^3 s}.

D8_CHAR_TABLE = {
    #        e   r2  r   s   rs
    "A1": (1, 1, 1, 1, 1),
    "A2": (1, 1, 1, -1, -1),
    "B1": (1, 1, -1, 1, -1),
    "B2": (1, 1, -1, -1, 1),
    "E": (2, -2, 0, 0, 0),
}


def d8_class(u):
    j, f = u
    if f == 0:
        return {0: 0, 2: 1, 1: 2, 3: 2}[j]
    return 3 if j % 2 == 0 else 4


def pin_d8_equivariance(forward, rng, elements, perm, F=3, T=4):
    """The linear layer commutes with every regular-action permutation."""
    x = rng.standard_normal((T, F, 8))
    ws = [rng.standard_normal((F, F)) for _ in range(4)] + [rng.standard_normal((2 * F, 2 * F))]
    y = forward(x, *ws)
    err = 0.0
    for u in elements:
        P = perm(u)
        lhs = forward(np.einsum("gh,tih->tig", P, x), *ws)
        rhs = np.einsum("gh,tih->tig", P, y)
        err = max(err, np.max(np.abs(lhs - rhs)))
    return err


def pin_d8_closed_forms(forward, rng, elements, slot, inv, mul, F=2):
    """Closed forms for one nonzero block at a time.

    A 1-D irrep chi with block w gives y[o,g] = chi(g)/8 sum_i w[o,i] sum_h chi(h) x[i,h].
    E with the identity block gives the isotypic projector
    y[i,g] = (2/8) sum_h chi_E(g h^-1) x[i,h].  All blocks identity gives y = x.
    """
    x = rng.standard_normal((3, F, 8))
    Z = np.zeros((F, F))
    ZE = np.zeros((2 * F, 2 * F))
    err = 0.0
    names = ("A1", "A2", "B1", "B2")
    for c, name in enumerate(names):
        w = rng.standard_normal((F, F))
        blocks = [Z, Z, Z, Z]
        blocks[c] = w
        chi = np.zeros(8)
        for u in elements:
            chi[slot(u)] = D8_CHAR_TABLE[name][d8_class(u)]
        ref = np.einsum("oi,g,tih,h->tog", w, chi, x, chi) / 8.0
        err = max(err, np.max(np.abs(forward(x, *blocks, ZE) - ref)))
    chiE = np.zeros((8, 8))
    for g in elements:
        for h in elements:
            chiE[slot(g), slot(h)] = D8_CHAR_TABLE["E"][d8_class(mul(g, inv(h)))]
    ref = np.einsum("gh,tih->tig", chiE, x) * (2.0 / 8.0)
    err = max(err, np.max(np.abs(forward(x, Z, Z, Z, Z, np.eye(2 * F)) - ref)))
    I = np.eye(F)
    err = max(err, np.max(np.abs(forward(x, I, I, I, I, np.eye(2 * F)) - x)))
    return err


def gelu_reference(v):
    """GELU(v) = v * Phi(v) with Phi from math.erf, element by element."""
    return np.vectorize(lambda t: 0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0))))(v)


# ---------------------------------------------------------------- backward pins


def brute_force_backward_data(dy, W):
    """dx[t,i,h] = sum_o sum_g W[o,i,(g-h) mod N] dy[t,o,g], by explicit loops."""
    T, Cout, N = dy.shape
    Cin = W.shape[1]
    dx = np.zeros((T, Cin, N))
    for t in range(T):
        for i in range(Cin):
            for h in range(N):
                s = 0.0
                for o in range(Cout):
                    for g in range(N):
                        s += float(W[o, i, (g - h) % N]) * float(dy[t, o, g])
                dx[t, i, h] = s
    return dx


def brute_force_weight_grad(x, dy):
    """dW[o,i,m] = sum_t sum_g dy[t,o,g] x[t,i,(g-m) mod N], by explicit loops."""
    T, Cin, N = x.shape
    Cout = dy.shape[1]
    dW = np.zeros((Cout, Cin, N))
    for o in range(Cout):
        for i in range(Cin):
            for m in range(N):
                s = 0.0
                for t in range(T):
                    for g in range(N):
                        s += float(dy[t, o, g]) * float(x[t, i, (g - m) % N])
                dW[o, i, m] = s
    return dW


_BWD_SHAPES = ((3, 2, 3, 1), (2, 3, 2, 2), (2, 2, 3, 3), (2, 3, 2, 4), (3, 2, 2, 5), (2, 2, 2, 8))


def pin_backward_data_bruteforce(backward_data, rng, shapes=_BWD_SHAPES):
    err = 0.0
    for T, Cin, Cout, N in shapes:
        dy = rng.standard_normal((T, Cout, N))
        W = rng.standard_normal((Cout, Cin, N))
        err = max(err, np.max(np.abs(backward_data(dy, W) - brute_force_backward_data(dy, W))))
    return err


def pin_weight_grad_bruteforce(weight_grad, rng, shapes=_BWD_SHAPES):
    err = 0.0
    for T, Cin, Cout, N in shapes:
        x = rng.standard_normal((T, Cin, N))
        dy = rng.standard_normal((T, Cout, N))
        err = max(err, np.max(np.abs(weight_grad(x, dy) - brute_force_weight_grad(x, dy))))
    return err


def pin_adjoint_identity(forward, backward_data, rng, shapes=((4, 3, 5, 4), (3, 2, 2, 8), (2, 5, 3, 7))):
    """<dx, u> = <dy, forward(u, W)> for every u: backward_data is the adjoint of
    the forward map (relative error of the two inner products)."""
    err = 0.0
    for T, Cin, Cout, N in shapes:
        u = rng.standard_normal((T, Cin, N))
        dy = rng.standard_normal((T, Cout, N))
        W = rng.standard_normal((Cout, Cin, N))
        a = float(np.sum(backward_data(dy, W) * u))
        b = float(np.sum(dy * forward(u, W)))
        err = max(err, abs(a - b) / max(abs(b), 1.0))
    return err


def pin_weight_grad_identity(forward, weight_grad, rng, shapes=((4, 3, 5, 4), (3, 2, 2, 8), (2, 5, 3, 7))):
    """y is linear in W, so <dW, V> = <dy, forward(x, V)> for every direction V
    (relative error of the two inner products)."""
    err = 0.0
    for T, Cin, Cout, N in shapes:
        x = rng.standard_normal((T, Cin, N))
        dy = rng.standard_normal((T, Cout, N))
        V = rng.standard_normal((Cout, Cin, N))
        a = float(np.sum(weight_grad(x, dy) * V))
        b = float(np.sum(dy * forward(x, V)))
        err = max(err, abs(a - b) / max(abs(b), 1.0))
    return err


def pin_weight_grad_fft(weight_grad, rng, Ns=(2, 3, 4, 8, 16)):
    """Cin = Cout = 1: dW is the token sum of the circular cross-correlation of
    dy with x, ifft(fft(dy) * conj(fft(x)))."""
    err = 0.0
    for N in Ns:
        x = rng.standard_normal((5, 1, N))
        dy = rng.standard_normal((5, 1, N))
        ref = np.real(np.fft.ifft(np.fft.fft(dy[:, 0, :], axis=-1) * np.conj(np.fft.fft(x[:, 0, :], axis=-1)),
                                  axis=-1)).sum(axis=0)
        err = max(err, np.max(np.abs(weight_grad(x, dy)[0, 0] - ref)))
    return err


def pin_backward_n1_matmul(backward_data, weight_grad, rng):
    """N = 1: dx = dy W and dW = dy^T x (plain matrix products)."""
    x = rng.standard_normal((6, 4, 1))
    dy = rng.standard_normal((6, 3, 1))
    W = rng.standard_normal((3, 4, 1))
    e1 = np.max(np.abs(backward_data(dy, W)[:, :, 0] - dy[:, :, 0] @ W[:, :, 0]))
    e2 = np.max(np.abs(weight_grad(x, dy)[:, :, 0] - dy[:, :, 0].T @ x[:, :, 0]))
    return float(max(e1, e2))
