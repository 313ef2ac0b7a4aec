"""CPU pins of the tensor-core weight packing's arithmetic.

cyclic_weight (where a layer's 8-slot weight V[o][i][m] comes from: the plain
weight, the backward data pass's adjoint, the two folds of a 16-slot weight
for the C_16 split, and their adjoints) and block_value (each entry of the
per-field spectral block matrix the MMAs multiply by) are host-and-device
functions in tc_pack_math.cuh.  A small host program compiled against that
header evaluates them on seeded bf16 weights; this test checks

  * cyclic_weight against each source's definition, exactly;
  * block_value semantically: with the forward transform F and the one-sided
    inverse I of the layer's coordinates, I . M . F applied to one field x
    must equal the layer on that field, the circular convolution
    y_g = sum_h V[(g - h) mod 8] x_h for the cyclic mode and the negacyclic
    one (the sign flips where the index wraps) for the negacyclic mode.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "tc_pack_math.cuh"
using namespace eqlin;
// stdin: mode wsrc F_in F_out n, then n weight values (bf16-representable)
int main() {
  int mode, wsrc, Fi, Fo, n;
  if (scanf("%d %d %d %d %d", &mode, &wsrc, &Fi, &Fo, &n) != 5) return 1;
  std::vector<__nv_bfloat16> W(n);
  for (int k = 0; k < n; ++k) { float v; scanf("%f", &v); W[k] = __float2bfloat16(v); }
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  if (mode == kModeCyclic4) {   // wsrc = adjoint flag; 4 slots
    for (int o = 0; o < Fo; ++o)
      for (int i = 0; i < Fi; ++i) {
        printf("V");
        for (int m = 0; m < 4; ++m) printf(" %.17g", c4_weight<false>(W.data(), Fi, Fo, wsrc, o, i, m));
        printf("\nM");
        for (int co = 0; co < 4; ++co)
          for (int ci = 0; ci < 4; ++ci)
            printf(" %.17g", c4_block_value<false>(W.data(), Fi, Fo, wsrc, co, o, ci, i));
        printf("\n");
      }
    return 0;
  }
  for (int o = 0; o < Fo; ++o)
    for (int i = 0; i < Fi; ++i) {
      printf("V");
      for (int m = 0; m < 8; ++m) printf(" %.17g", cyclic_weight<false>(W.data(), Fi, Fo, wsrc, o, i, m));
      printf("\nM");
      for (int co = 0; co < 8; ++co)
        for (int ci = 0; ci < 8; ++ci) {
          const double v = mode == kModeCyclic8
                               ? block_value<kModeCyclic8, false>(W.data(), none, Fi, Fo, wsrc, co, o, ci, i)
                               : block_value<kModeNegacyclic8, false>(W.data(), none, Fi, Fo, wsrc, co, o, ci, i);
          printf(" %.17g", v);
        }
      printf("\n");
    }
  return 0;
}
"""

WSRC = {"plain": 0, "adjoint": 1, "fold_even": 2, "fold_odd": 3, "fold_even_adj": 4, "fold_odd_adj": 5}


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("pk")
    src = d / "pk.cu"
    src.write_text(HARNESS)
    exe = d / "pk"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-o", str(exe), str(src)], check=True, capture_output=True)
    return str(exe)


def run(exe, mode, wsrc, Fi, Fo, W):
    flat = W.reshape(-1)
    inp = f"{mode} {WSRC[wsrc]} {Fi} {Fo} {flat.size}\n" + " ".join(repr(float(v)) for v in flat) + "\n"
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout.splitlines()
    V = np.array([[float(t) for t in l.split()[1:]] for l in out if l.startswith("V")]).reshape(Fo, Fi, 8)
    M = np.array([[float(t) for t in l.split()[1:]] for l in out if l.startswith("M")]).reshape(Fo, Fi, 8, 8)
    return V, M


def weights(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).double().numpy()


def expected_V(W, wsrc, o, i):
    m = np.arange(8)
    if wsrc == "plain":
        return W[o, i, m]
    if wsrc == "adjoint":
        return W[i, o, (-m) % 8]
    if wsrc in ("fold_even", "fold_odd"):
        a, b = W[o, i, m], W[o, i, m + 8]
    else:
        a, b = W[i, o, (16 - m) % 16], W[i, o, (16 - (m + 8)) % 16]
    return 0.5 * (a + b) if wsrc.startswith("fold_even") else 0.5 * (a - b)


def cyclic_F_I():
    h = np.arange(8)
    F = np.zeros((8, 8))
    F[0] = 1.0
    F[7] = (-1.0) ** h
    for k in range(1, 4):
        F[2 * k - 1] = np.cos(2 * np.pi * h * k / 8)
        F[2 * k] = -np.sin(2 * np.pi * h * k / 8)
    I = np.zeros((8, 8))
    I[:, 0] = 1.0
    I[:, 7] = (-1.0) ** h
    for k in range(1, 4):
        I[:, 2 * k - 1] = np.cos(2 * np.pi * h * k / 8)
        I[:, 2 * k] = -np.sin(2 * np.pi * h * k / 8)
    mask = np.zeros((8, 8), bool)
    mask[0, 0] = mask[7, 7] = True
    for k in range(1, 4):
        mask[2 * k - 1:2 * k + 1, 2 * k - 1:2 * k + 1] = True
    return F, I, mask


def negacyclic_F_I():
    h = np.arange(8)
    F = np.zeros((8, 8))
    I = np.zeros((8, 8))
    mask = np.zeros((8, 8), bool)
    for b in range(4):
        ph = np.pi * h * (2 * b + 1) / 8
        F[2 * b], F[2 * b + 1] = np.cos(ph), -np.sin(ph)
        I[:, 2 * b], I[:, 2 * b + 1] = np.cos(ph), -np.sin(ph)
        mask[2 * b:2 * b + 2, 2 * b:2 * b + 2] = True
    return F, I, mask


def layer_on_one_field(V, x, negacyclic):
    y = np.zeros(8)
    for g in range(8):
        for h in range(8):
            s = -1.0 if (negacyclic and h > g) else 1.0
            y[g] += s * V[(g - h) % 8] * x[h]
    return y


@pytest.mark.parametrize("wsrc", list(WSRC))
def test_weight_sources(harness, wsrc):
    Fi, Fo = 3, 2
    slots = 8 if wsrc in ("plain", "adjoint") else 16
    shape = (Fo, Fi, slots) if "adj" not in wsrc else (Fi, Fo, slots)
    W = weights(shape, seed=WSRC[wsrc])
    V, _ = run(harness, 0, wsrc, Fi, Fo, W)
    for o in range(Fo):
        for i in range(Fi):
            assert np.array_equal(V[o, i], expected_V(W, wsrc, o, i)), (o, i)


@pytest.mark.parametrize("mode", [0, 2])
@pytest.mark.parametrize("wsrc", ["plain", "adjoint", "fold_odd"])
def test_block_matrix_reproduces_the_layer_on_one_field(harness, mode, wsrc):
    Fi, Fo = 2, 3
    slots = 8 if wsrc in ("plain", "adjoint") else 16
    shape = (Fo, Fi, slots) if "adj" not in wsrc else (Fi, Fo, slots)
    W = weights(shape, seed=10 + mode)
    V, M = run(harness, mode, wsrc, Fi, Fo, W)
    F, I, mask = negacyclic_F_I() if mode == 2 else cyclic_F_I()
    x = np.random.default_rng(mode).standard_normal(8)
    for o in range(Fo):
        for i in range(Fi):
            got = I @ (np.where(mask, M[o, i], 0.0) @ (F @ x))
            want = layer_on_one_field(V[o, i], x, negacyclic=(mode == 2))
            assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want))), (o, i)


def test_negacyclic_field_layer_is_the_oracles():
    """The one-field negacyclic layer used above agrees with the oracle's."""
    rng = np.random.default_rng(3)
    V = rng.standard_normal(8)
    x = rng.standard_normal(8)
    want = oracle.negacyclic_forward(x.reshape(1, 1, 8), V.reshape(1, 1, 8))[0, 0]
    assert np.allclose(layer_on_one_field(V, x, negacyclic=True), want, atol=1e-12)


@pytest.mark.parametrize("adjoint", [0, 1])
def test_c4_block_matrix_reproduces_the_layer_on_one_field(harness, adjoint):
    """p4: with F = [Re X0; Re X1; Im X1; Re X2] rows and the one-sided inverse
    I (bin 1 already doubled), I . M . F on one field is the 4-slot circular
    convolution with V (the plain weight, or the adjoint W[i][o][(-m) mod 4])."""
    Fi, Fo = 3, 2
    shape = (Fo, Fi, 4) if not adjoint else (Fi, Fo, 4)
    W = weights(shape, seed=20 + adjoint)
    flat = W.reshape(-1)
    inp = f"3 {adjoint} {Fi} {Fo} {flat.size}\n" + " ".join(repr(float(v)) for v in flat) + "\n"
    out = subprocess.run([harness], input=inp, capture_output=True, text=True, check=True).stdout.splitlines()
    V = np.array([[float(t) for t in l.split()[1:]] for l in out if l.startswith("V")]).reshape(Fo, Fi, 4)
    M = np.array([[float(t) for t in l.split()[1:]] for l in out if l.startswith("M")]).reshape(Fo, Fi, 4, 4)
    h = np.arange(4)
    F = np.stack([np.ones(4), np.cos(np.pi * h / 2), -np.sin(np.pi * h / 2), (-1.0) ** h])
    I = np.stack([np.ones(4), np.cos(np.pi * h / 2), -np.sin(np.pi * h / 2), (-1.0) ** h], axis=1)
    mask = np.zeros((4, 4), bool)
    mask[0, 0] = mask[3, 3] = True
    mask[1:3, 1:3] = True
    x = np.random.default_rng(adjoint).standard_normal(4)
    for o in range(Fo):
        for i in range(Fi):
            want_V = W[i, o, (-np.arange(4)) % 4] if adjoint else W[o, i]
            assert np.array_equal(V[o, i], want_V)
            got = I @ (np.where(mask, M[o, i], 0.0) @ (F @ x))
            want = np.array([sum(want_V[(g - hh) % 4] * x[hh] for hh in range(4)) for g in range(4)])
            assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))
