"""CPU emulation of the tensor-core weight gradient's data layout (C_8).

The kernel's result rests on several index rules agreeing with one another:
where the producer's TMA boxes (128-byte swizzle) put each (token, field)
of dy and x, where the in-place transform writes each spectral coordinate,
how the MMA descriptors (K-major, no swizzle, leading/stride byte offsets)
address those coordinates as operands, the MMA list (parsed from the kernel
source), the pair instruction's TMEM layout, and which (split, o, i,
coordinate) each epilogue thread stores.  This test restates each rule in
numpy on an fp64 model of shared memory and TMEM (unwritten cells are NaN),
runs the units of the token splits, applies the fixed-order reduction and
inverse transform the CUDA-core path uses, and requires the fp64 oracle's
weight gradient to rounding.  It checks the layout, not the hardware: the GPU
tests check the hardware.
"""

import math
import os
import re

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc", "wgrad_tc.cu")


def _src():
    return open(SRC).read()


def _const(name):
    m = re.search(r"constexpr (?:int|uint32_t) %s = (\d+);" % name, _src())
    assert m, name
    return int(m.group(1))


def mma_list():
    """(ca, cb, g, neg) in issue order, from the kernel's wt_mma switch."""
    src = _src()
    body = src[src.index("constexpr WtMma wt_mma(int f) {"):]
    body = body[: body.index("default:")]
    cases = re.findall(r"case (\d+): return \{([-\d, ]+)\};", body)
    return [tuple(int(v) for v in vals.split(",")) for _, vals in sorted(cases, key=lambda c: int(c[0]))]


TK = _const("kWtTk")
PAIRS = _const("kWtPairs")
OTILE = _const("kWtOTile")
ITILE = _const("kWtITile")
SUB = _const("kWtSub")
EPI0 = _const("kWtEpi0")
ATOMS = TK // 8
BOX = TK * 128
HALF = 8 * BOX
STAGE = 2 * HALF


def plan(T, Cin, Cout):
    n_ot = -(-Cout // OTILE)
    n_it = -(-Cin // ITILE)
    ntile = n_ot * n_it
    if T <= 0:
        return n_it, ntile, 0, TK
    target = PAIRS if ntile <= 4 else -(-4 * PAIRS // ntile)
    tps = -(-T // target)
    tps = -(-tps // TK) * TK
    return n_it, ntile, -(-T // tps), tps


def half_spectrum(v):
    """[..., 8] -> [..., 8]: Re X0, Re X1, Im X1, Re X2, Im X2, Re X3, Im X3, Re X4,
    X_k = sum_h v_h exp(-2 pi i h k / 8)."""
    X = np.fft.fft(v, axis=-1)
    return np.stack([X[..., 0].real, X[..., 1].real, X[..., 1].imag, X[..., 2].real,
                     X[..., 2].imag, X[..., 3].real, X[..., 3].imag, X[..., 4].real], axis=-1)


def inverse_matrix():
    """dW[m] = (1/8) sum_c Inv[m][c] C_c (one-sided inverse of the half spectrum)."""
    inv = np.zeros((8, 8))
    for m in range(8):
        inv[m, 0] = 1.0
        inv[m, 7] = (-1.0) ** m
        for k in range(1, 4):
            th = 2 * math.pi * m * k / 8
            inv[m, 2 * k - 1] = 2 * math.cos(th)
            inv[m, 2 * k] = -2 * math.sin(th)
    return inv


def tma_box(smem, off, src, field0, tok):
    """One box: TK token rows of 8 fields x 8 bf16 (128 bytes), 128-byte swizzle;
    out-of-range tokens or fields read as zero."""
    T, F, _ = src.shape
    for r in range(TK):
        t = tok + r
        for f in range(8):
            val = src[t, field0 + f] if (t < T and field0 + f < F) else np.zeros(8)
            chunk = f ^ (r % 8)
            start = (off + r * 128 + chunk * 16) // 2
            smem[start:start + 8] = val


def transform_atom(smem, atom):
    """Read the 1 KB atom whole (8 token rows, swizzled), write coordinate c of
    (token row r, field f) at atom + 128 c + 16 f + 2 r."""
    v = np.empty((8, 8, 8))
    for r in range(8):
        for f in range(8):
            start = (atom + r * 128 + ((f ^ r) * 16)) // 2
            v[r, f] = smem[start:start + 8]
    z = half_spectrum(v)
    for r in range(8):
        for f in range(8):
            for c in range(8):
                smem[(atom + c * 128 + f * 16 + r * 2) // 2] = z[r, f, c]


def operand(smem, start, rows):
    """K-major, no swizzle: element (m, k) of a 16-wide K-step at
    start + (m // 8) SBO + (k // 8) LBO + 16 (m % 8) + 2 (k % 8), LBO = 1 KB, SBO = one box."""
    out = np.empty((rows, 16))
    for m in range(rows):
        for k in range(16):
            out[m, k] = smem[(start + (m // 8) * BOX + (k // 8) * 1024 + (m % 8) * 16 + (k % 8) * 2) // 2]
    return out


def emulate(x, dy):
    T, Cin, _ = x.shape
    Cout = dy.shape[1]
    n_it, ntile, S, tps = plan(T, Cin, Cout)
    mmas = mma_list()
    part = np.full((S, Cout, Cin, 8), np.nan)
    for u in range(S * ntile):
        s, tile = divmod(u, ntile)
        ot, it = divmod(tile, n_it)
        nsub = 2 if Cin - it * ITILE > SUB else 1
        tmem = [np.full((128, 512), np.nan) for _ in range(2)]
        t0 = s * tps
        t1 = min(T, t0 + tps)
        for ch in range(-(-(t1 - t0) // TK)):
            tok = t0 + ch * TK
            smem = [np.full(STAGE // 2, np.nan) for _ in range(2)]
            for r in range(2):
                # producer
                for b in range(8):
                    tma_box(smem[r], b * BOX, dy, ot * OTILE + r * 64 + 8 * b, tok)
                for b in range(8):
                    fi = it * ITILE + (b >> 2) * SUB + r * 32 + 8 * (b & 3)
                    tma_box(smem[r], HALF + b * BOX, x, fi, tok)
                # in-place transform (boxes past the fields are skipped: zero stays zero)
                for j in range(16 * ATOMS):
                    which = j // (8 * ATOMS)
                    b, a = (j // ATOMS) % 8, j % ATOMS
                    field0 = (ot * OTILE + r * 64 + 8 * b if which == 0
                              else it * ITILE + (b >> 2) * SUB + r * 32 + 8 * (b & 3))
                    if field0 >= (Cout if which == 0 else Cin):
                        continue
                    transform_atom(smem[r], which * HALF + b * BOX + a * 1024)
            # MMAs: pair instruction M = 128 (64 rows per CTA), N = 64 nsub (32 nsub B rows
            # per CTA: its x boxes from the first), coordinate group g at TMEM columns 64 g
            nb = 32 * nsub
            for ks in range(TK // 16):
                acc = ch > 0 or ks > 0
                for f, (ca, cb, g, neg) in enumerate(mmas):
                    accf = acc or any(mmas[e][2] == g for e in range(f))
                    A = np.vstack([operand(smem[r], ca * 128 + ks * 2048, 64) for r in range(2)])
                    B = np.vstack([operand(smem[r], HALF + cb * 128 + ks * 2048, nb) for r in range(2)])
                    D = A @ B.T * (-1.0 if neg else 1.0)
                    col = g * 64
                    for r in range(2):
                        Dr = D[64 * r: 64 * r + 64]
                        blk = np.vstack([Dr[:, :nb], Dr[:, nb:]])   # lanes 64.. hold columns N/2..
                        tmem[r][:, col:col + nb] = blk + (tmem[r][:, col:col + nb] if accf else 0.0)
        # epilogue: warps EPI0..EPI0+7, 16x256b loads
        for r in range(2):
            for w in range(8):
                q4, sub = (EPI0 + w) & 3, w >> 2
                h = q4 >> 1
                for lane in range(32):
                    tq, tr = lane & 3, lane >> 2
                    o0 = ot * OTILE + r * 64 + (q4 & 1) * 32 + sub * 16 + tr
                    for st in range(nsub):
                        for fg in range(0, 32, 8):
                            i0 = it * ITILE + st * SUB + h * 32 + fg + 2 * tq
                            for e in range(4):
                                o, i = o0 + 8 * (e >> 1), i0 + (e & 1)
                                tl = q4 * 32 + sub * 16 + tr + 8 * (e >> 1)
                                tc = fg + 2 * tq + (e & 1)
                                if o < Cout and i < Cin:
                                    assert np.all(np.isnan(part[s, o, i])), "written twice"
                                    part[s, o, i] = [tmem[r][tl, c * 64 + st * 32 + tc] for c in range(8)]
    assert not np.isnan(part).any(), "a partial was never written or read an unwritten cell"
    C = part.sum(axis=0)
    return np.einsum("mc,oic->oim", inverse_matrix(), C) / 8.0


@pytest.mark.parametrize("T,Cin,Cout", [(40, 24, 16), (70, 136, 40), (33, 8, 136),
                                         # a subtile of one field; 129 fields: a second tile of one
                                         (32, 65, 8), (31, 129, 64), (64, 128, 129)])
def test_tensor_core_weight_gradient_layout_reproduces_the_oracle(T, Cin, Cout):
    x, _W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, 8, torch.float64, seed=5)
    x, dy = x.numpy(), dy.numpy()
    got = emulate(x, dy)
    want = oracle.cyclic_weight_grad(x, dy)
    assert np.max(np.abs(got - want)) <= 1e-11 * max(1.0, np.max(np.abs(want)))


def test_mma_list_covers_every_bin_product():
    """Per bin: Re C = DYr Xr + DYi Xi, Im C = DYi Xr - DYr Xi; real bins one product."""
    terms = {}
    for ca, cb, g, neg in mma_list():
        terms.setdefault(g, set()).add((ca, cb, -1 if neg else 1))
    assert terms[0] == {(0, 0, 1)} and terms[7] == {(7, 7, 1)}
    for k in range(1, 4):
        re_, im_ = 2 * k - 1, 2 * k
        assert terms[re_] == {(re_, re_, 1), (im_, im_, 1)}
        assert terms[im_] == {(im_, re_, 1), (re_, im_, -1)}


def test_split_plan_covers_the_tokens_once():
    for T, Cin, Cout in [(1, 1, 1), (31, 8, 8), (131072, 160, 160), (65536, 96, 384), (8192, 64, 64)]:
        n_it, ntile, S, tps = plan(T, Cin, Cout)
        assert tps % TK == 0 and S * tps >= T and (S - 1) * tps < T
        assert S <= max(PAIRS, 4 * PAIRS)
