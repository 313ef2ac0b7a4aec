"""Plain fp64 CPU oracle for the equivariant linear layers.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA library and imports nothing from it.

Everything here is written for a reader checking it against the source pages
by eye: no blocking, no fusion, no transform beyond what the definition states.
All arithmetic is float64; inputs are widened to float64 on entry, so when the
GPU receives bf16 values the oracle sees exactly those values.

Two layers:

* Cyclic EQ-Linear over C_N in the regular representation.  The layer is the
  naive "replicate the shared weight into a dense matrix and multiply" form
  (Flash EQ-Linear, gist.science/paper/2607.21271, Technical Summary >
  Problem Statement; the group-circulant weight of Methodology > Core Insight):

      y[t, o, g] = sum_i sum_h W[o, i, (g - h) mod N] * x[t, i, h]

  The dense (Cout*N) x (Cin*N) matrix is built explicitly and applied.  The
  oracle never uses a DFT: the fast path's Fourier route is what it checks.

* D8 Fourier-domain linear layer (Quick ViTs, papernotes.org ECCV2026 review,
  "Key design 1" and "Key design 2").  The steps are taken in the page's
  order: change of basis from the regular representation to the irreps
  A1, A2, B1, B2 and 2 x E; four (C/8)-square block products and one
  (C/4)-square product shared by E's two row coordinates; the change of basis
  back; optionally an exact-erf GELU in the regular domain.  The page's
  formulas for the basis are lost in extraction, so the concrete basis below
  is a stated reading (see the D8 section).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force and library routines (numpy FFT,
numpy matmul, math.erf) -- none of which reuse this module's arithmetic.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

# ---------------------------------------------------------------------------
# Cyclic group C_N
# ---------------------------------------------------------------------------


def cyclic_dense_matrix(W: np.ndarray) -> np.ndarray:
    """Expand the shared weight W[o, i, m] (m in Z_N) into the dense matrix.

    Wd[o*N + g, i*N + h] = W[o, i, (g - h) mod N]   (block (g, h) of the
    group-circulant matrix; Flash EQ-Linear, Methodology > Core Insight).
    Returns float64 of shape (Cout*N, Cin*N).
    """
    W = np.asarray(W, dtype=np.float64)
    Cout, Cin, N = W.shape
    g = np.arange(N)[:, None]
    h = np.arange(N)[None, :]
    m = (g - h) % N                      # m[g, h] = (g - h) mod N
    blocks = W[:, :, m]                  # [o, i, g, h] = W[o, i, (g-h) mod N]
    dense = blocks.transpose(0, 2, 1, 3)  # [o, g, i, h]
    return np.ascontiguousarray(dense.reshape(Cout * N, Cin * N))


def cyclic_forward(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Naive EQ-Linear: y[t] = Wd @ x[t] with the dense expanded matrix.

    x: [T, Cin, N], W: [Cout, Cin, N]  ->  y: [T, Cout, N], float64.
    (Flash EQ-Linear, Technical Summary > Problem Statement: the
    replicate-and-dense-multiply baseline, applied here in fp64.)
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    T, Cin, N = x.shape
    Cout, Cin_w, N_w = W.shape
    if Cin_w != Cin or N_w != N:
        raise ValueError("x and W disagree on Cin or N")
    Wd = cyclic_dense_matrix(W)
    y = x.reshape(T, Cin * N) @ Wd.T
    return y.reshape(T, Cout, N)


def cyclic_backward_data(dy: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Gradient with respect to x of sum(dy * y), y = cyclic_forward(x, W).

    The layer is the linear map y[t] = Wd @ x[t] with the dense expanded
    matrix, so the gradient is its transpose applied to dy:
        dx[t] = Wd^T @ dy[t].
    dy: [T, Cout, N], W: [Cout, Cin, N]  ->  dx: [T, Cin, N], float64.
    (The backward pass of the same layer: Flash EQ-Linear, Technical Summary,
    where the Fourier route also serves backpropagation.)
    """
    dy = np.asarray(dy, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    T, Cout, N = dy.shape
    Cout_w, Cin, N_w = W.shape
    if Cout_w != Cout or N_w != N:
        raise ValueError("dy and W disagree on Cout or N")
    Wd = cyclic_dense_matrix(W)
    dx = dy.reshape(T, Cout * N) @ Wd
    return dx.reshape(T, Cin, N)


def cyclic_weight_grad(x: np.ndarray, dy: np.ndarray) -> np.ndarray:
    """Gradient with respect to the shared weight W of sum(dy * y).

    Every dense entry Wd[o*N + g, i*N + h] with (g - h) mod N = m is a copy of
    the one shared parameter W[o, i, m] (Flash EQ-Linear, Methodology > Core
    Insight), so its gradient is the sum of the dense-matrix gradient
        G[o*N + g, i*N + h] = sum_t dy[t, o, g] * x[t, i, h]
    over those copies.
    x: [T, Cin, N], dy: [T, Cout, N]  ->  dW: [Cout, Cin, N], float64.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    T, Cin, N = x.shape
    T_d, Cout, N_d = dy.shape
    if T_d != T or N_d != N:
        raise ValueError("x and dy disagree on T or N")
    G = (dy.reshape(T, Cout * N).T @ x.reshape(T, Cin * N)).reshape(Cout, N, Cin, N)
    dW = np.zeros((Cout, Cin, N))
    for g in range(N):
        for h in range(N):
            dW[:, :, (g - h) % N] += G[:, g, :, h]
    return dW


def negacyclic_forward(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Negacyclic counterpart of the layer (product modulo z^N + 1 instead of z^N - 1):

        y[t, o, g] = sum_i sum_h s(g, h) W[o, i, (g - h) mod N] x[t, i, h],
        s(g, h) = +1 if h <= g, -1 if h > g (the index wrapped around).

    Not a layer of the pages: with it, C_2N splits into a C_N cyclic and a C_N
    negacyclic layer on the sums and differences of the two halves of the group
    axis (X(z) mod z^2N - 1 = (z^N - 1)(z^N + 1)), which the tests pin.
    x: [T, Cin, N], W: [Cout, Cin, N]  ->  y: [T, Cout, N], float64, through the
    dense signed matrix.
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    T, Cin, N = x.shape
    Cout = W.shape[0]
    g = np.arange(N)[:, None]
    h = np.arange(N)[None, :]
    sign = np.where(h <= g, 1.0, -1.0)                       # [g, h]
    blocks = W[:, :, (g - h) % N] * sign[None, None]         # [o, i, g, h]
    Wd = blocks.transpose(0, 2, 1, 3).reshape(Cout * N, Cin * N)
    return (x.reshape(T, Cin * N) @ Wd.T).reshape(T, Cout, N)


def cyclic_counts(N: int, Cin: int, Cout: int) -> dict:
    """Parameter and multiply counts of the cyclic layer, per token.

    Dense form: (Cout*N) x (Cin*N) multiplies.  Fourier form (Flash EQ-Linear,
    Algorithmic Approach > Conjugate Symmetry, Specialization for p4): a real
    input has a half spectrum; bin 0 (and bin N/2 for even N) is real and
    costs one real Cin x Cout product, every other kept bin is complex and
    costs four.  Parameters: Cout*Cin*N shared weights against the dense
    matrix's (Cout*N)*(Cin*N).
    """
    kept = N // 2 + 1
    real_bins = 2 if N % 2 == 0 and N > 1 else 1
    complex_bins = kept - real_bins
    real_products = real_bins + 4 * complex_bins
    return {
        "kept_bins": kept,
        "real_bins": real_bins,
        "complex_bins": complex_bins,
        "real_gemms": real_products,
        "dense_gemms": N * N,
        "dense_macs": N * N * Cin * Cout,
        "fourier_macs": real_products * Cin * Cout,
        "params": Cout * Cin * N,
        "dense_params": (Cout * N) * (Cin * N),
    }


# ---------------------------------------------------------------------------
# Dihedral group D8 (order 8): rotations r^j and reflections r^j s
# ---------------------------------------------------------------------------
#
# Reading (the page's equations for the group and basis are lost):
#   D8 = <r, s | r^4 = s^2 = 1, s r s = r^-1>.  Element (j, f) means r^j s^f.
#   Regular slot order: slot j <-> r^j (j = 0..3), slot 4 + j <-> r^j s.
#   Regular action (left): (u . x)(g) = x(u^-1 g), a permutation of slots.
#   Irreps: A1: r->1, s->1;  A2: r->1, s->-1;  B1: r->-1, s->1;
#           B2: r->-1, s->-1;  E: r->[[0,-1],[1,0]], s->[[1,0],[0,-1]].
#   Fourier coordinates per field, in order
#           [A1, A2, B1, B2, E00, E01, E10, E11]   (E_ab, a = row, b = column)
#   with Q[chi, g] = chi(g)/sqrt(8) for the 1-D irreps and
#        Q[E_ab, g] = rho_E(g)[a, b] * sqrt(2/8).
#   Weights: wA1, wA2, wB1, wB2 are [C/8, C/8] ([out, in]); wE is [C/4, C/4]
#   acting on the vector v_a[e] with e = 2*i + b (field i, column b), once
#   for each row a in {0, 1} with the same matrix.

D8_ORDER = 8
D8_COORDS = ("A1", "A2", "B1", "B2", "E00", "E01", "E10", "E11")


def d8_elements() -> list:
    """The 8 elements as (j, f) = r^j s^f in regular-slot order."""
    return [(j, 0) for j in range(4)] + [(j, 1) for j in range(4)]


def d8_mul(u: tuple, v: tuple) -> tuple:
    """(r^j1 s^f1)(r^j2 s^f2) = r^(j1 + (-1)^f1 j2) s^(f1 + f2), from s r = r^-1 s."""
    j1, f1 = u
    j2, f2 = v
    sign = -1 if f1 else 1
    return ((j1 + sign * j2) % 4, (f1 + f2) % 2)


def d8_inv(u: tuple) -> tuple:
    for v in d8_elements():
        if d8_mul(u, v) == (0, 0):
            return v
    raise AssertionError("no inverse")


def d8_slot(u: tuple) -> int:
    return d8_elements().index(u)


def d8_regular_perm(u: tuple) -> np.ndarray:
    """8x8 permutation P_u of the left regular action: (P_u x)[g] = x[u^-1 g]."""
    P = np.zeros((8, 8))
    ui = d8_inv(u)
    for g in d8_elements():
        P[d8_slot(g), d8_slot(d8_mul(ui, g))] = 1.0
    return P


def d8_rho_E(u: tuple) -> np.ndarray:
    """2-D irrep E: rho(r) = rotation by 90 degrees, rho(s) = diag(1, -1)."""
    R = np.array([[0.0, -1.0], [1.0, 0.0]])
    S = np.array([[1.0, 0.0], [0.0, -1.0]])
    j, f = u
    return np.linalg.matrix_power(R, j) @ np.linalg.matrix_power(S, f)


def d8_chars_1d(u: tuple) -> np.ndarray:
    """Values of A1, A2, B1, B2 at u = r^j s^f."""
    j, f = u
    return np.array([1.0, (-1.0) ** f, (-1.0) ** j, (-1.0) ** (j + f)])


def d8_Q() -> np.ndarray:
    """8x8 change of basis, regular slots -> [A1, A2, B1, B2, E00, E01, E10, E11]."""
    Q = np.zeros((8, 8))
    for g in d8_elements():
        s = d8_slot(g)
        Q[0:4, s] = d8_chars_1d(g) / math.sqrt(8.0)
        rho = d8_rho_E(g)
        for a in range(2):
            for b in range(2):
                Q[4 + 2 * a + b, s] = rho[a, b] * math.sqrt(2.0 / 8.0)
    return Q


def gelu_exact(v: np.ndarray) -> np.ndarray:
    """GELU(v) = 0.5 v (1 + erf(v / sqrt 2)), the exact (erf) form, in fp64."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + _erf(v / math.sqrt(2.0)))


def d8_forward(x, wA1, wA2, wB1, wB2, wE, fuse_gelu: bool = False) -> np.ndarray:
    """D8 Fourier-domain linear layer, steps in the page's order.

    x: [T, F, 8] with F = C/8 fields in the regular representation.
    wA1..wB2: [F, F]; wE: [2F, 2F] ([out, in], y = W @ v).
    Returns y: [T, F, 8] float64 (GELU applied in the regular domain if asked).
    (Quick ViTs review, Key design 1: channels as 8-dim Fourier reps;
    Key design 2: Schur blocks, E shared over two coordinates, GELU only in
    the regular domain where the group acts by permutation.)
    """
    x = np.asarray(x, dtype=np.float64)
    T, F, eight = x.shape
    if eight != 8:
        raise ValueError("last axis must be the 8 regular slots")
    Q = d8_Q()
    # 1. change of basis, per field: z[t, i, :] = Q x[t, i, :]
    z = np.einsum("cg,tig->tic", Q, x)
    zo = np.zeros_like(z)
    # 2a. four (C/8)-square blocks on the 1-D irreps
    for c, w in enumerate((wA1, wA2, wB1, wB2)):
        w = np.asarray(w, dtype=np.float64)
        zo[:, :, c] = z[:, :, c] @ w.T
    # 2b. the (C/4)-square E block, once per row coordinate a
    wE = np.asarray(wE, dtype=np.float64)
    for a in range(2):
        v = np.empty((T, 2 * F))
        for b in range(2):
            v[:, b::2] = z[:, :, 4 + 2 * a + b]      # v[e = 2i + b]
        vo = v @ wE.T
        for b in range(2):
            zo[:, :, 4 + 2 * a + b] = vo[:, b::2]
    # 3. back to the regular representation: x' = Q^T z'
    y = np.einsum("cg,tic->tig", Q, zo)
    # 4. optional GELU in the regular domain
    if fuse_gelu:
        y = gelu_exact(y)
    return y


def d8_dense_operator(wA1, wA2, wB1, wB2, wE) -> np.ndarray:
    """The C x C regular-domain matrix of the (linear part of the) D8 layer.

    Built column by column by pushing basis vectors through ``d8_forward``;
    used by the pins (equivariance, group-convolution structure, rank).
    Index [o*8 + g, i*8 + h].
    """
    F = np.asarray(wA1).shape[0]
    C = 8 * F
    eye = np.eye(C).reshape(C, F, 8)
    cols = d8_forward(eye, wA1, wA2, wB1, wB2, wE, fuse_gelu=False)
    return cols.reshape(C, C).T


def d8_counts(C: int) -> dict:
    """Parameters and multiplies per token of a C -> C layer (Quick ViTs,
    Key design 2): dense C^2 against four (C/8)^2 blocks plus one (C/4)^2 block
    stored once but applied to both E row coordinates."""
    if C % 8:
        raise ValueError("C must be a multiple of 8")
    F = C // 8
    params = 4 * F * F + (2 * F) ** 2
    mults = 4 * F * F + 2 * (2 * F) ** 2
    return {"dense_params": C * C, "params": params,
            "dense_mults": C * C, "mults": mults,
            "param_ratio": C * C / params, "mult_ratio": C * C / mults}


# ---------------------------------------------------------------------------
# D8 MLP block kept in the Fourier domain
# ---------------------------------------------------------------------------


def d8_fourier_linear(z, wA1, wA2, wB1, wB2, wE) -> np.ndarray:
    """D8 equivariant linear map acting on Fourier coordinates, F_in -> F_out fields.

    z: [T, F_in, 8] per field in the order [A1, A2, B1, B2, E00, E01, E10, E11];
    wA1..wB2: [F_out, F_in]; wE: [2 F_out, 2 F_in] acting on the vector
    v_a[e = 2i + b] = z[:, i, E_ab] for each row coordinate a, the same matrix for
    a = 0 and a = 1.  Returns [T, F_out, 8].
    (Quick ViTs review, Key design 1: features stay in the Fourier domain between
    layers; Key design 2: the Schur blocks, E shared over its two row
    coordinates; the MLP's C -> 4C expansion and 4C -> C contraction are the
    rectangular case.)
    """
    z = np.asarray(z, dtype=np.float64)
    T, F_in, eight = z.shape
    if eight != 8:
        raise ValueError("last axis must hold the 8 Fourier coordinates")
    F_out = np.asarray(wA1).shape[0]
    zo = np.zeros((T, F_out, 8))
    for c, w in enumerate((wA1, wA2, wB1, wB2)):
        zo[:, :, c] = z[:, :, c] @ np.asarray(w, dtype=np.float64).T
    wE = np.asarray(wE, dtype=np.float64)
    for a in range(2):
        v = np.empty((T, 2 * F_in))
        for b in range(2):
            v[:, b::2] = z[:, :, 4 + 2 * a + b]
        vo = v @ wE.T
        for b in range(2):
            zo[:, :, 4 + 2 * a + b] = vo[:, b::2]
    return zo


def d8_gelu_roundtrip(z) -> np.ndarray:
    """Fourier coordinates -> regular domain -> exact GELU -> Fourier coordinates,
    per field: Q GELU(Q^T z).  (Quick ViTs review, Key design 2: the pointwise
    nonlinearity is applied in the regular domain, where the group acts by
    permuting slots, so it stays equivariant.)"""
    Q = d8_Q()
    x = np.einsum("cg,tic->tig", Q, np.asarray(z, dtype=np.float64))
    return np.einsum("cg,tig->tic", Q, gelu_exact(x))


def d8_mlp_block(z, w1, w2) -> np.ndarray:
    """The transformer MLP kept in the Fourier domain: expand with the blocks w1
    (F -> F_hidden), GELU round trip, contract with the blocks w2 (F_hidden -> F).
    w1, w2: tuples (wA1, wA2, wB1, wB2, wE) as for d8_fourier_linear."""
    return d8_fourier_linear(d8_gelu_roundtrip(d8_fourier_linear(z, *w1)), *w2)


# ---------------------------------------------------------------------------
# Error measure shared by the tests
# ---------------------------------------------------------------------------


def rel_frobenius(a, b) -> float:
    """||a - b||_F / ||b||_F in float64 (b is the oracle); ||a||_F when b is all zero.

    Pinned by tests/test_oracle_metric.py (hand values, normalisation by b,
    exact rational brute force)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    num = np.linalg.norm((a - b).ravel())
    return float(num / den) if den > 0 else float(num)
