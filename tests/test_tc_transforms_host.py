"""CPU pins of the tensor-core kernels' per-field transforms.

The transforms in tc_transforms.cuh are host-and-device inline functions (the
device build uses sm_100's paired fp32 instructions, a host build the scalar
operations, which round the same way).  This test compiles a small host
program against that header (nvcc, no GPU needed), runs every transform on
seeded inputs and compares it with its definition in numpy, so a wrong sign,
index or twiddle fails here rather than as a parity failure on a GPU:

  fwd_cyclic8      [Re X0, Re X1, Im X1, Re X2, Im X2, Re X3, Im X3, Re X4],
                   X_k = sum_h x_h e^{-2 pi i h k / 8}
  inv_cyclic8      y_g = Y0 + (-1)^g Y4 + sum_{k=1..3} Re(Y'_k e^{2 pi i g k / 8})
                   (the complex bins Y' already doubled)
  fwd_negacyclic8  [Re D_b, Im D_b] for b = 0..3, D_b = sum_h d_h e^{-i pi h (2b+1) / 8}
  inv_negacyclic8  y_g = sum_{b=0..3} Re(Y_b e^{i pi g (2b+1) / 8})
  fwd_d8, inv_d8   z = Q x and x = Q^T z with the oracle's D8 change of basis Q
  gelu_erf2        GELU(v) = v Phi(v) within the stated 3e-6
  gelu_tanh2       GELU(v) within 4.8e-4 (the tanh form's own deviation; the
                   host build uses tanhf, the device's tanh.approx adds at most
                   0.5 |v| 2^-11, bounded separately below)
"""

import math
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <cstring>
#include "tc_transforms.cuh"
using namespace eqlin;
typedef void (*Fn)(const float2 (&)[8], float2 (&)[8]);
int main(int argc, char **argv) {
  Fn fn = nullptr;
  const char *name = argv[1];
  if (!strcmp(name, "fwd_cyclic8")) fn = fwd_cyclic8;
  if (!strcmp(name, "inv_cyclic8")) fn = inv_cyclic8;
  if (!strcmp(name, "fwd_negacyclic8")) fn = fwd_negacyclic8;
  if (!strcmp(name, "inv_negacyclic8")) fn = inv_negacyclic8;
  if (!strcmp(name, "fwd_d8")) fn = fwd_d8;
  if (!strcmp(name, "inv_d8")) fn = inv_d8;
  if (!strcmp(name, "fwd_cyclic4x2")) fn = fwd_cyclic4x2;
  if (!strcmp(name, "inv_cyclic4x2")) fn = inv_cyclic4x2;
  float a[8], b[8];
  for (;;) {
    for (int i = 0; i < 8; ++i) if (scanf("%f", &a[i]) != 1) return 0;
    for (int i = 0; i < 8; ++i) if (scanf("%f", &b[i]) != 1) return 0;
    float2 x[8], z[8];
    for (int i = 0; i < 8; ++i) x[i] = make_float2(a[i], b[i]);
    if (fn) {
      fn(x, z);
    } else if (!strcmp(name, "gelu_tanh")) {   // lane-wise
      for (int i = 0; i < 8; ++i) z[i] = gelu_tanh2(x[i]);
    } else {   // gelu_erf2, lane-wise
      for (int i = 0; i < 8; ++i) z[i] = gelu_erf2(x[i]);
    }
    for (int i = 0; i < 8; ++i) printf("%.9g ", z[i].x);
    for (int i = 0; i < 8; ++i) printf("%.9g ", z[i].y);
    printf("\n");
  }
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("tx")
    src = d / "tx.cu"
    src.write_text(HARNESS)
    exe = d / "tx"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-o", str(exe), str(src)], check=True, capture_output=True)
    return str(exe)


def run(exe, name, rows):
    """rows: [n, 8]; pairs of rows go in as the two float2 lanes."""
    assert len(rows) % 2 == 0
    inp = "\n".join(" ".join(repr(float(v)) for v in r) for r in rows) + "\n"
    out = subprocess.run([exe, name], input=inp, capture_output=True, text=True, check=True).stdout
    a = np.array([[float(t) for t in line.split()] for line in out.strip().splitlines()])
    return np.concatenate([a[:, :8], a[:, 8:]], axis=0), np.concatenate([rows[0::2], rows[1::2]], axis=0)


def _rows(seed, n=64):
    return np.random.default_rng(seed).standard_normal((n, 8)).astype(np.float32).astype(np.float64)


def _check(got, want, tol=3e-6):
    assert np.max(np.abs(got - want)) <= tol * max(1.0, np.max(np.abs(want)))


def test_fwd_cyclic8(harness):
    got, x = run(harness, "fwd_cyclic8", _rows(1))
    X = np.fft.fft(x, axis=-1)
    want = np.stack([X[:, 0].real, X[:, 1].real, X[:, 1].imag, X[:, 2].real, X[:, 2].imag,
                     X[:, 3].real, X[:, 3].imag, X[:, 4].real], axis=-1)
    _check(got, want)


def test_inv_cyclic8(harness):
    got, z = run(harness, "inv_cyclic8", _rows(2))
    g = np.arange(8)
    want = z[:, [0]] + ((-1.0) ** g)[None, :] * z[:, [7]]
    for k in range(1, 4):
        th = 2 * np.pi * g * k / 8
        want = want + z[:, [2 * k - 1]] * np.cos(th)[None, :] - z[:, [2 * k]] * np.sin(th)[None, :]
    _check(got, want)


def test_fwd_negacyclic8(harness):
    got, d = run(harness, "fwd_negacyclic8", _rows(3))
    h = np.arange(8)
    want = np.empty_like(d)
    for b in range(4):
        D = (d * np.exp(-1j * np.pi * h * (2 * b + 1) / 8)[None, :]).sum(axis=1)
        want[:, 2 * b], want[:, 2 * b + 1] = D.real, D.imag
    _check(got, want)


def test_inv_negacyclic8(harness):
    got, z = run(harness, "inv_negacyclic8", _rows(4))
    g = np.arange(8)
    want = np.zeros_like(z)
    for b in range(4):
        Y = z[:, [2 * b]] + 1j * z[:, [2 * b + 1]]
        want += (Y * np.exp(1j * np.pi * g * (2 * b + 1) / 8)[None, :]).real
    _check(got, want)


def test_negacyclic_round_trip_is_the_negacyclic_identity(harness):
    """inv(fwd(d)) = 4 d (the one-sided inverse's 2/8 lives in the weights)."""
    d = _rows(5)
    z, _ = run(harness, "fwd_negacyclic8", d)
    # run() returned the lanes in [first rows of pairs; second rows] order
    zz = np.empty_like(z)
    n = len(d) // 2
    zz[0::2], zz[1::2] = z[:n], z[n:]
    y, _ = run(harness, "inv_negacyclic8", zz)
    _check(y, 4 * np.concatenate([d[0::2], d[1::2]], axis=0), tol=1e-5)


def test_d8_basis_is_the_oracles(harness):
    Q = oracle.d8_Q()
    got, x = run(harness, "fwd_d8", _rows(6))
    _check(got, x @ Q.T)
    got, z = run(harness, "inv_d8", _rows(7))
    _check(got, z @ Q)


def test_gelu_erf2_within_its_bound(harness):
    v = np.linspace(-6, 6, 128).reshape(16, 8).astype(np.float32).astype(np.float64)
    got, v2 = run(harness, "gelu", v)
    erf = np.vectorize(math.erf)
    want = 0.5 * v2 * (1 + erf(v2 / math.sqrt(2)))
    assert np.max(np.abs(got - want)) <= 3e-6 * max(1.0, np.max(np.abs(v2)))


def test_gelu_tanh2_within_its_bound(harness):
    v = np.linspace(-10, 10, 4096).reshape(512, 8).astype(np.float32).astype(np.float64)
    got, v2 = run(harness, "gelu_tanh", v)
    erf = np.vectorize(math.erf)
    want = 0.5 * v2 * (1 + erf(v2 / math.sqrt(2)))
    err = np.abs(got - want)
    assert np.max(err) <= 4.8e-4 + 2e-7 * np.max(np.abs(v2)), np.max(err)
    # the form itself, in float64 with an exact tanh: its deviation peaks near |v| = 2.7
    vv = np.linspace(-10, 10, 200001)
    form = 0.5 * vv * (1 + np.tanh(math.sqrt(2 / math.pi) * (vv + 0.044715 * vv ** 3)))
    exact = 0.5 * vv * (1 + erf(vv / math.sqrt(2)))
    assert 4.5e-4 < np.max(np.abs(form - exact)) <= 4.8e-4
    # a hardware tanh with relative error 2^-11 moves GELU by at most 0.5 |v| 2^-11,
    # under half a bf16 unit (2^-9 relative) wherever |GELU(v)| >= |v| / 4
    assert 0.5 * 2.0 ** -11 < 0.25 * 2.0 ** -9


F16_HARNESS = r"""
#include <cstdio>
#include <cstring>
#include "tc_transforms.cuh"
using namespace eqlin;
// stdin: 16 fp16 bit patterns (two 16-byte chunks a, b); prints the 8 float2
// of unpack_f16x8_pair, then pack_f16x2 of each float2 as a 32-bit word
int main() {
  unsigned v[16];
  for (;;) {
    for (int i = 0; i < 16; ++i) if (scanf("%u", &v[i]) != 1) return 0;
    uint32_t w[8];
    for (int k = 0; k < 8; ++k) w[k] = v[2 * k] | (v[2 * k + 1] << 16);
    uint4 a = make_uint4(w[0], w[1], w[2], w[3]), b = make_uint4(w[4], w[5], w[6], w[7]);
    float2 f[8];
    unpack_f16x8_pair(a, b, f);
    for (int i = 0; i < 8; ++i) printf("%.17g %.17g ", f[i].x, f[i].y);
    for (int i = 0; i < 8; ++i) printf("%u ", pack_f16x2(f[i].x * 1.0001f, f[i].y));
    printf("\n");
  }
}
"""


@pytest.fixture(scope="module")
def f16_harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("f16")
    src = d / "f16.cu"
    src.write_text(F16_HARNESS)
    exe = d / "f16"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-o", str(exe), str(src)], check=True, capture_output=True)
    return str(exe)


def test_fp16_unpack_lane_order_and_pack_rounding(f16_harness):
    """Chunk a holds fp16 values a0..a7, chunk b holds b0..b7 (element j at
    bytes 2j): unpack must give f[j] = (a_j, b_j), the layout the transforms
    read; pack_f16x2(lo, hi) must round each to nearest fp16 with lo in the
    low half."""
    rng = np.random.default_rng(0)
    vals = rng.standard_normal((32, 16)).astype(np.float16)
    bits = vals.view(np.uint16).astype(np.uint32)
    inp = "\n".join(" ".join(str(int(b)) for b in row) for row in bits) + "\n"
    out = subprocess.run([f16_harness], input=inp, capture_output=True, text=True, check=True).stdout
    for row, line in zip(vals, out.strip().splitlines()):
        t = line.split()
        f = np.array([float(x) for x in t[:16]]).reshape(8, 2)
        assert np.array_equal(f[:, 0], row[:8].astype(np.float64))     # lane x: chunk a
        assert np.array_equal(f[:, 1], row[8:].astype(np.float64))     # lane y: chunk b
        words = np.array([int(x) for x in t[16:]], dtype=np.uint32)
        lo = (words & 0xFFFF).astype(np.uint16).view(np.float16)
        hi = (words >> 16).astype(np.uint16).view(np.float16)
        assert np.array_equal(lo, (row[:8].astype(np.float32) * np.float32(1.0001)).astype(np.float16))
        assert np.array_equal(hi, row[8:])


def test_p4_super_field_transforms(harness):
    """Each 8-slot super-field is two C_4 fields: fwd gives [Re X0, Re X1, Im X1,
    Re X2] per field, X_k = sum_h x_h e^{-2 pi i h k / 4}; inv gives
    y_g = Y0 + (-1)^g Y2 + Re(Y'_1 i^g) with Y'_1 already doubled."""
    got, x = run(harness, "fwd_cyclic4x2", _rows(8))
    X = np.fft.fft(x.reshape(-1, 2, 4), axis=-1)
    want = np.stack([X[..., 0].real, X[..., 1].real, X[..., 1].imag, X[..., 2].real], axis=-1).reshape(-1, 8)
    _check(got, want)
    got, z = run(harness, "inv_cyclic4x2", _rows(9))
    zz = z.reshape(-1, 2, 4)
    g = np.arange(4)
    want = (zz[..., 0:1] + ((-1.0) ** g) * zz[..., 3:4] + zz[..., 1:2] * np.cos(np.pi * g / 2)
            - zz[..., 2:3] * np.sin(np.pi * g / 2)).reshape(-1, 8)
    _check(got, want)
