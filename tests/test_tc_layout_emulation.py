"""CPU emulation of the tensor-core path's data layout for the cyclic C_8 layer.

The fused kernel's correctness rests on several tables agreeing with one
another: where the weight packer puts each spectrum value, the MMA list the
issuer walks (A coordinate, weight panel, starting row, leading byte offset,
N, negate-B, overwrite-or-accumulate), where the transform puts each
coordinate of x, and which coordinate each TMEM column group holds for the
inverse transform.  This test restates those rules in numpy, runs the MMA
list in fp64 with the MMA's arithmetic (D = A . B^T per instruction), and
requires the result to equal the dense fp64 oracle to rounding.  The MMA
list itself is parsed from the kernel source, so the test follows the table
the kernel uses.  The GPU tests check the same path on the hardware; this one
runs anywhere and fails on an inconsistent refactor of the layout.
"""

import os
import re

import numpy as np
import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "group_wise_dft_b200", "csrc", "spectral_tc.cu")

K_CO_MAX = 64
NUM_PANELS = 5                      # cyclic: W0, W4, bins 1..3 as [Wi; Wr]
GROUP_COORD = [0, 7, 2, 1, 4, 3, 6, 5]


def _source():
    return open(SRC).read()


def ks_full():
    m = re.search(r"#define EQLIN_KS_FULL (\d+)", _source())
    return int(m.group(1))


def mma_list():
    """The cyclic MMA list in issue order: (blk, pair, panel, dgroup, wide, neg, roff)."""
    src = _source()
    body = src[src.index("constexpr MmaDesc mma_desc(int mode, int i, int m) {"):]
    body = body[: body.index("default:")]
    cases = re.findall(r"case (\d+): return \{([-\d, ]+)\};", body)
    return [tuple(int(v) for v in vals.split(",")) for _, vals in sorted(cases, key=lambda c: int(c[0]))]


def chunk_fields(Fo, c):
    return min(K_CO_MAX, Fo - c * K_CO_MAX)


def num_chunks(Fo):
    return (Fo + K_CO_MAX - 1) // K_CO_MAX


def panel_bytes(k, co):
    return 16 * co if k < 2 else 32 * co


def panel_offset(k, co):
    return sum(panel_bytes(i, co) for i in range(k))


def stage_bytes(co):
    return panel_offset(NUM_PANELS, co)


def panel_rows(k, co):
    return panel_bytes(k, co) // 32


def chunk_ks(Fi, Fo, c):
    nst = Fi // 16
    ks = 2 * ks_full() if 2 * chunk_fields(Fo, c) <= K_CO_MAX else ks_full()
    while ks > 1 and nst % ks:
        ks //= 2
    return ks


def stage_offset(Fi, Fo, c, jp, h):
    full = 2 * (Fi // 16) * stage_bytes(K_CO_MAX)
    ks = chunk_ks(Fi, Fo, c)
    s, q = divmod(jp, ks)
    return c * full + ((2 * s + h) * ks + q) * stage_bytes(chunk_fields(Fo, c))


def spectrum_entry(W, cout, o, cin, i):
    """Block-matrix value: output coordinate cout of field o from input coordinate
    cin of field i; coordinates [Re0, Re1, Im1, Re2, Im2, Re3, Im3, Re4]; the 1/8 and
    the one-sided inverse's 2 folded in."""
    b = 0 if cout == 0 else (4 if cout == 7 else (cout + 1) // 2)
    m = np.arange(8)
    ang = 2 * np.pi * ((m * b) % 8) / 8
    re = np.sum(W[o, i] * np.cos(ang)) / 8
    im = -np.sum(W[o, i] * np.sin(ang)) / 8
    if b in (0, 4):
        return re
    out_re, in_re = (cout & 1) == 1, (cin & 1) == 1
    return 2 * ((re if in_re else -im) if out_re else (im if in_re else re))


def pack(W, Fi, Fo, entry=None):
    """The packed weight buffer, in bf16 elements (held as fp64).  entry(cout, o,
    cin, i) gives each value (default: the layer's spectral block entries)."""
    if entry is None:
        entry = lambda co_, o_, ci_, i_: spectrum_entry(W, co_, o_, ci_, i_)
    total = stage_offset(Fi, Fo, num_chunks(Fo) - 1, Fi // 16, 0)
    B = np.full(total // 2, np.nan)
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        for jp in range(Fi // 16):
            for hh in range(2):
                off = stage_offset(Fi, Fo, c, jp, hh) // 2
                for e in range(stage_bytes(co) // 2):
                    k = 0
                    while k + 1 < NUM_PANELS and 2 * e >= panel_offset(k + 1, co):
                        k += 1
                    w = e - panel_offset(k, co) // 2
                    if k < 2:
                        kc, r, el = w // (hc * 8), (w // 8) % hc, w % 8
                        o, i = c * K_CO_MAX + hh * hc + r, (2 * jp + kc) * 8 + el
                        cr = 0 if k == 0 else 7
                        val = entry(cr, o, cr, i)
                    else:
                        kc, r, el = w // (co * 8), (w // 8) % co, w % 8
                        o, i = c * K_CO_MAX + hh * hc + (r % hc), (2 * jp + kc) * 8 + el
                        b = k - 1
                        cre, cim = 2 * b - 1, 2 * b
                        val = entry(cim, o, cre, i) if r < hc else entry(cre, o, cre, i)
                    assert np.isnan(B[off + e]), "two panel elements packed to one place"
                    B[off + e] = val
    assert not np.any(np.isnan(B)), "packed buffer has holes"
    return B


def x_coordinates(x):
    """[T, F, 8] -> [T, F, 8] real half-spectrum coordinates [Re0, Re1, Im1, .., Re4]."""
    X = np.fft.fft(x, axis=-1)
    return np.stack([X[..., 0].real, X[..., 1].real, X[..., 1].imag, X[..., 2].real, X[..., 2].imag,
                     X[..., 3].real, X[..., 3].imag, X[..., 4].real], axis=-1)


def inverse(Y):
    """y_g = Y0 + (-1)^g Y4 + sum_k (Re Y_k cos - Im Y_k sin)(2 pi g k / 8); Y's complex bins
    already carry the factor 2 and all of it the 1/8."""
    g = np.arange(8)
    y = Y[..., 0:1] + ((-1.0) ** g) * Y[..., 7:8]
    for k in (1, 2, 3):
        th = 2 * np.pi * g * k / 8
        y = y + Y[..., 2 * k - 1:2 * k] * np.cos(th) - Y[..., 2 * k:2 * k + 1] * np.sin(th)
    return y


def emulate(x, W, Z=None, B=None):
    """x [T, Fi, 8] -> y through the C_8 layout; Z (coordinates, [T, Fi, 8]) and
    B (the packed weights) may be given instead of being derived from x and W."""
    T, Fi, _ = (x.shape if Z is None else Z.shape)
    Fo = W.shape[0]
    B = pack(W, Fi, Fo) if B is None else B
    Z = x_coordinates(x) if Z is None else Z               # [T, Fi, 8]
    mmas = mma_list()
    acc_first = []
    for f, (_, _, _, dg, _, _, _) in enumerate(mmas):
        acc_first.append(any(dg >= e[3] and dg < e[3] + 1 + e[4] for e in mmas[:f]))
    y = np.zeros((T, Fo, 8))
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        ks = chunk_ks(Fi, Fo, c)
        # two CTA halves of B; D per half: [T, 8 groups * hc columns]
        D = [np.full((T, 8 * hc), np.nan) for _ in range(2)]
        for jp in range(Fi // 16):
            s, q = divmod(jp, ks)
            assert stage_offset(Fi, Fo, c, jp, 0) == stage_offset(Fi, Fo, c, s * ks, 0) + q * stage_bytes(co)
            for f, (blk, pair, panel, dgroup, wide, neg, roff) in enumerate(mmas):
                A = Z[:, 16 * jp:16 * jp + 16, 4 * blk + pair]         # [T, K = 16 fields]
                rows = co if wide else hc
                lbo = panel_rows(panel, co) * 16
                for h in range(2):
                    start = stage_offset(Fi, Fo, c, jp, h) + panel_offset(panel, co) + roff * hc * 16
                    n = np.arange(rows)[:, None]
                    k = np.arange(16)[None, :]
                    byte = start + (n // 8) * 128 + (n % 8) * 16 + (k // 8) * lbo + (k % 8) * 2
                    assert np.all(byte < stage_offset(Fi, Fo, c, jp, h) + stage_bytes(co)), "B read past its stage"
                    Bm = B[byte // 2]                                # [rows, 16]
                    prod = (A @ Bm.T) * (-1.0 if neg else 1.0)       # [T, rows]
                    cols = slice(dgroup * hc, dgroup * hc + rows)
                    if jp == 0 and not acc_first[f]:
                        D[h][:, cols] = prod
                    else:
                        D[h][:, cols] = D[h][:, cols] + prod
        for h in range(2):
            assert not np.any(np.isnan(D[h])), "a TMEM column group was never written"
            Y = np.zeros((T, hc, 8))
            for kk in range(8):
                Y[:, :, GROUP_COORD[kk]] = D[h][:, kk * hc:(kk + 1) * hc]
            y[:, c * K_CO_MAX + h * hc:c * K_CO_MAX + (h + 1) * hc, :] = inverse(Y)
    return y


@pytest.mark.parametrize("Fi,Fo", [(32, 96), (48, 64), (64, 32), (16, 160)])
def test_tensor_core_layout_reproduces_the_layer(Fi, Fo):
    rng = np.random.default_rng(Fi + Fo)
    x = rng.standard_normal((6, Fi, 8))
    W = rng.standard_normal((Fo, Fi, 8)) / np.sqrt(8 * Fi)
    y = emulate(x, W)
    ref = oracle.cyclic_forward(x, W)
    assert oracle.rel_frobenius(y, ref) < 1e-12


def test_mma_list_is_parsed():
    mmas = mma_list()
    assert len(mmas) == 11 and all(len(m) == 7 for m in mmas)


# ------------------------------------------------------------------ D8

# The D8 MMA list in issue order (lists 0..3, two MMAs each):
#   A1 | A2, B1 | B2 (N = co), then E row a = 0 and a = 1 for the K-steps of
#   blocks 2jp and 2jp+1 (N = 2co: output rows (b', field)), both rows a
#   reading the same E panel.
D8_MMAS = [(0, 0, 0, 0, 0, 0, 0), (0, 1, 1, 1, 0, 0, 0), (1, 0, 2, 2, 0, 0, 0), (1, 1, 3, 3, 0, 0, 0),
           (0, 2, 4, 4, 1, 0, 0), (1, 2, 5, 4, 1, 0, 0), (0, 3, 4, 6, 1, 0, 0), (1, 3, 5, 6, 1, 0, 0)]


def test_d8_mma_list_matches_the_kernel_source():
    src = _source()
    body = src[src.index("constexpr MmaDesc mma_desc(int mode, int i, int m) {"):]
    body = body[body.index("  switch (i) {"):body.index("\n}\n")]
    found = re.findall(r"MmaDesc\{([^}]*)\}", body)
    expect = ["0, 0, 0, 0, 0, 0, 0", "0, 1, 1, 1, 0, 0, 0", "1, 0, 2, 2, 0, 0, 0", "1, 1, 3, 3, 0, 0, 0",
              "m, 2, 4 + m, 4, 1, 0, 0", "m, 3, 4 + m, 6, 1, 0, 0"]
    assert found == expect


def d8_panel_bytes(k, co):
    return 16 * co if k < 4 else 32 * co


def d8_panel_offset(k, co):
    return sum(d8_panel_bytes(i, co) for i in range(k))


def d8_stage_offset(Fi, Fo, c, jp, h):
    sb = lambda co: d8_panel_offset(6, co)
    full = 2 * (Fi // 16) * sb(K_CO_MAX)
    ks = chunk_ks(Fi, Fo, c)
    s, q = divmod(jp, ks)
    return c * full + ((2 * s + h) * ks + q) * sb(chunk_fields(Fo, c))


def d8_pack(ws, wE, Fi, Fo):
    """ws[k]: [Fo, Fi]; wE: [2 Fo, 2 Fi] (rows e' = 2o + b', columns e = 2i + b)."""
    sb = lambda co: d8_panel_offset(6, co)
    total = d8_stage_offset(Fi, Fo, num_chunks(Fo) - 1, Fi // 16, 0)
    B = np.full(total // 2, np.nan)
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        for jp in range(Fi // 16):
            for hh in range(2):
                off = d8_stage_offset(Fi, Fo, c, jp, hh) // 2
                for e in range(sb(co) // 2):
                    k = 0
                    while k + 1 < 6 and 2 * e >= d8_panel_offset(k + 1, co):
                        k += 1
                    w = e - d8_panel_offset(k, co) // 2
                    if k < 4:
                        kc, r, el = w // (hc * 8), (w // 8) % hc, w % 8
                        o, i = c * K_CO_MAX + hh * hc + r, (2 * jp + kc) * 8 + el
                        val = ws[k][o, i]
                    else:
                        kstep = 2 * jp + (k - 4)
                        kc, r, el = w // (co * 8), (w // 8) % co, w % 8
                        bo = 1 if r >= hc else 0
                        o, i = c * K_CO_MAX + hh * hc + (r % hc), kstep * 8 + el
                        val = wE[2 * o + bo, 2 * i + kc]
                    B[off + e] = val
    assert not np.any(np.isnan(B))
    return B


def d8_emulate(x, ws, wE, in_fourier=False, out="regular"):
    """The fused kernel's D8 mode.  x: [T, Fi, 8] regular slots, or coordinates
    if in_fourier (the transform only places them); out: "regular" (Q^T),
    "fourier" (coordinates as accumulated) or "roundtrip" (Q GELU(Q^T .))."""
    T, Fi, _ = x.shape
    Fo = ws[0].shape[0]
    F = Fi
    Q = oracle.d8_Q()
    Z = x if in_fourier else np.einsum("cg,tig->tic", Q, x)   # [T, Fi, 8] coordinates
    B = d8_pack(ws, wE, Fi, Fo)
    acc_first = [any(m[3] >= e[3] and m[3] < e[3] + 1 + e[4] for e in D8_MMAS[:f])
                 for f, m in enumerate(D8_MMAS)]
    y = np.zeros((T, Fo, 8))
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        D = [np.full((T, 8 * hc), np.nan) for _ in range(2)]
        for jp in range(F // 16):
            for f, (blk, pair, panel, dgroup, wide, neg, roff) in enumerate(D8_MMAS):
                if pair < 2:          # A1, A2 (row 0) or B1, B2 (row 1): 16 fields of one coordinate
                    A = Z[:, 16 * jp:16 * jp + 16, 2 * blk + pair]
                else:                 # E row a = pair - 2 of block 2jp + blk: (b = 0, b = 1) x 8 fields
                    a = pair - 2
                    fl = slice(8 * (2 * jp + blk), 8 * (2 * jp + blk) + 8)
                    A = np.concatenate([Z[:, fl, 4 + 2 * a], Z[:, fl, 4 + 2 * a + 1]], axis=1)
                rows = co if wide else hc
                lbo = (d8_panel_bytes(panel, co) // 32) * 16
                for h in range(2):
                    start = d8_stage_offset(Fi, Fo, c, jp, h) + d8_panel_offset(panel, co) + roff * hc * 16
                    n = np.arange(rows)[:, None]
                    k = np.arange(16)[None, :]
                    Bm = B[(start + (n // 8) * 128 + (n % 8) * 16 + (k // 8) * lbo + (k % 8) * 2) // 2]
                    prod = (A @ Bm.T) * (-1.0 if neg else 1.0)
                    cols = slice(dgroup * hc, dgroup * hc + rows)
                    if jp == 0 and not acc_first[f]:
                        D[h][:, cols] = prod
                    else:
                        D[h][:, cols] = D[h][:, cols] + prod
        for h in range(2):
            assert not np.any(np.isnan(D[h]))
            Zo = np.stack([D[h][:, kk * hc:(kk + 1) * hc] for kk in range(8)], axis=-1)   # group k = coordinate k
            if out == "fourier":
                Yo = Zo
            else:
                Yo = np.einsum("cg,tic->tig", Q, Zo)
                if out == "roundtrip":
                    Yo = np.einsum("cg,tig->tic", Q, oracle.gelu_exact(Yo))
            y[:, c * K_CO_MAX + h * hc:c * K_CO_MAX + (h + 1) * hc, :] = Yo
    return y


@pytest.mark.parametrize("C", [256, 512, 768])
def test_d8_tensor_core_layout_reproduces_the_layer(C):
    F = C // 8
    rng = np.random.default_rng(C)
    x = rng.standard_normal((5, F, 8))
    ws = [rng.standard_normal((F, F)) / np.sqrt(C) for _ in range(4)]
    wE = rng.standard_normal((2 * F, 2 * F)) / np.sqrt(C)
    y = d8_emulate(x, ws, wE)
    ref = oracle.d8_forward(x, *ws, wE, fuse_gelu=False)
    assert oracle.rel_frobenius(y, ref) < 1e-12


@pytest.mark.parametrize("Fi,Fo", [(160, 640), (32, 96), (48, 32)])
@pytest.mark.parametrize("out", ["fourier", "roundtrip"])
def test_d8_fourier_domain_layer_layout(Fi, Fo, out):
    """Rectangular Fourier-domain layer (input already coordinates, output as
    coordinates or through the GELU round trip) against the oracle."""
    rng = np.random.default_rng(Fi + Fo)
    z = rng.standard_normal((3, Fi, 8))
    s = 1.0 / np.sqrt(8 * Fi)
    ws = [rng.standard_normal((Fo, Fi)) * s for _ in range(4)]
    wE = rng.standard_normal((2 * Fo, 2 * Fi)) * s
    y = d8_emulate(z, ws, wE, in_fourier=True, out=out)
    ref = oracle.d8_fourier_linear(z, *ws, wE)
    if out == "roundtrip":
        ref = oracle.d8_gelu_roundtrip(ref)
    assert oracle.rel_frobenius(y, ref) < 1e-12


@pytest.mark.parametrize("Fi,Fo,gelu", [(640, 32, True), (176, 64, False), (352, 96, True)])
def test_d8_fourier_column_slices_reproduce_the_wide_layer(Fi, Fo, gelu):
    """A layer wider than the resident A operand runs as column slices of at
    most 160 input fields: slice s packs the blocks' columns [160 s, 160 s + w)
    (E's columns [320 s, 320 s + 2w), e = 2i + b), reads the same columns of z,
    writes a partial; the partials are summed, then the round trip if asked."""
    rng = np.random.default_rng(Fi + Fo)
    z = rng.standard_normal((3, Fi, 8))
    s = 1.0 / np.sqrt(8 * Fi)
    ws = [rng.standard_normal((Fo, Fi)) * s for _ in range(4)]
    wE = rng.standard_normal((2 * Fo, 2 * Fi)) * s
    total = np.zeros((3, Fo, 8))
    for k0 in range(0, Fi, 160):
        k1 = min(Fi, k0 + 160)
        total += d8_emulate(z[:, k0:k1], [w[:, k0:k1] for w in ws], wE[:, 2 * k0:2 * k1],
                            in_fourier=True, out="fourier")
    if gelu:
        total = oracle.d8_gelu_roundtrip(total)
    ref = oracle.d8_fourier_linear(z, *ws, wE)
    if gelu:
        ref = oracle.d8_gelu_roundtrip(ref)
    assert oracle.rel_frobenius(total, ref) < 1e-12


# ------------------------------------------------------------------ C_16 in two passes


def neg_mma_list():
    """The negacyclic MMA list in issue order, parsed from the kernel source."""
    src = _source()
    body = src[src.index("constexpr MmaDesc mma_desc(int mode, int i, int m) {"):]
    body = body[body.index("if (mode == kModeNegacyclic8) {"):]
    body = body[: body.index("default:")]
    cases = re.findall(r"case (\d+): return \{([-\d, ]+)\};", body)
    return [tuple(int(v) for v in vals.split(",")) for _, vals in sorted(cases, key=lambda c: int(c[0]))]


def neg_coordinates(d):
    """[T, F, 8] -> [Re D0, Im D0, .., Re D3, Im D3], D_b = sum_h d_h e^{-i pi h (2b+1) / 8}."""
    h = np.arange(8)
    out = []
    for b in range(4):
        ang = np.pi * h * (2 * b + 1) / 8
        out += [np.sum(d * np.cos(ang), axis=-1), -np.sum(d * np.sin(ang), axis=-1)]
    return np.stack(out, axis=-1)


def neg_inverse(Y):
    g = np.arange(8)
    y = np.zeros(Y.shape[:-1] + (8,))
    for b in range(4):
        th = np.pi * g * (2 * b + 1) / 8
        y = y + Y[..., 2 * b:2 * b + 1] * np.cos(th) - Y[..., 2 * b + 1:2 * b + 2] * np.sin(th)
    return y


def neg_entry(W, cout, o, cin, i):
    """Negacyclic block-matrix value (coordinates [Re, Im] per bin, 2/8 folded in)."""
    b = cout >> 1
    m = np.arange(8)
    ang = np.pi * ((m * (2 * b + 1)) % 16) / 8
    re = 2 * np.sum(W[o, i] * np.cos(ang)) / 8
    im = -2 * np.sum(W[o, i] * np.sin(ang)) / 8
    out_re, in_re = (cout & 1) == 0, (cin & 1) == 0
    return (re if in_re else -im) if out_re else (im if in_re else re)


def neg_emulate(d, W8):
    """The negacyclic mode: all four panels are combined [Wi; Wr] panels (bin b = panel b)."""
    T, Fi, _ = d.shape
    Fo = W8.shape[0]
    nst = Fi // 16
    # stage layout of this mode: 4 panels of 32 co bytes = 128 co, as in the cyclic mode
    B = np.full(stage_offset(Fi, Fo, num_chunks(Fo) - 1, nst, 0) // 2, np.nan)
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        for jp in range(nst):
            for hh in range(2):
                off = stage_offset(Fi, Fo, c, jp, hh) // 2
                for e in range(128 * co // 2):
                    k, w = divmod(e, 16 * co)
                    kc, r, el = w // (co * 8), (w // 8) % co, w % 8
                    o, i = c * K_CO_MAX + hh * hc + (r % hc), (2 * jp + kc) * 8 + el
                    cre, cim = 2 * k, 2 * k + 1
                    B[off + e] = neg_entry(W8, cim, o, cre, i) if r < hc else neg_entry(W8, cre, o, cre, i)
    assert not np.any(np.isnan(B))
    Z = neg_coordinates(d)
    mmas = neg_mma_list()
    acc_first = [any(m[3] >= e[3] and m[3] < e[3] + 1 + e[4] for e in mmas[:f]) for f, m in enumerate(mmas)]
    y = np.zeros((T, Fo, 8))
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        D = [np.full((T, 8 * hc), np.nan) for _ in range(2)]
        for jp in range(nst):
            for f, (blk, pair, panel, dgroup, wide, neg, roff) in enumerate(mmas):
                A = Z[:, 16 * jp:16 * jp + 16, 4 * blk + pair]
                rows = co if wide else hc
                for h in range(2):
                    start = stage_offset(Fi, Fo, c, jp, h) + panel * 32 * co + roff * hc * 16
                    n = np.arange(rows)[:, None]
                    k = np.arange(16)[None, :]
                    Bm = B[(start + (n // 8) * 128 + (n % 8) * 16 + (k // 8) * (co * 16) + (k % 8) * 2) // 2]
                    prod = (A @ Bm.T) * (-1.0 if neg else 1.0)
                    cols = slice(dgroup * hc, dgroup * hc + rows)
                    if jp == 0 and not acc_first[f]:
                        D[h][:, cols] = prod
                    else:
                        D[h][:, cols] = D[h][:, cols] + prod
        for h in range(2):
            assert not np.any(np.isnan(D[h]))
            Y = np.zeros((T, hc, 8))
            for kk in range(8):
                Y[:, :, kk ^ 1] = D[h][:, kk * hc:(kk + 1) * hc]     # group k holds coordinate k ^ 1
            y[:, c * K_CO_MAX + h * hc:c * K_CO_MAX + (h + 1) * hc, :] = neg_inverse(Y)
    return y


def test_negacyclic_mma_list_is_parsed():
    mmas = neg_mma_list()
    assert len(mmas) == 12 and all(len(m) == 7 for m in mmas)


@pytest.mark.parametrize("Fi,Fo", [(32, 96), (16, 64), (48, 32)])
def test_negacyclic_layout_reproduces_the_negacyclic_layer(Fi, Fo):
    rng = np.random.default_rng(Fi * 7 + Fo)
    d = rng.standard_normal((5, Fi, 8))
    W8 = rng.standard_normal((Fo, Fi, 8)) / np.sqrt(8 * Fi)
    ref = oracle.negacyclic_forward(d, W8)
    assert oracle.rel_frobenius(neg_emulate(d, W8), ref) < 1e-12


@pytest.mark.parametrize("Fi,Fo", [(32, 96), (16, 32)])
def test_c16_two_pass_reproduces_the_c16_layer(Fi, Fo):
    rng = np.random.default_rng(Fi + 3 * Fo)
    x = rng.standard_normal((4, Fi, 16))
    W = rng.standard_normal((Fo, Fi, 16)) / np.sqrt(16 * Fi)
    e, d = x[..., :8] + x[..., 8:], x[..., :8] - x[..., 8:]
    ye = emulate(e, 0.5 * (W[..., :8] + W[..., 8:]))          # the cyclic mode, even fold (halved)
    yo = neg_emulate(d, 0.5 * (W[..., :8] - W[..., 8:]))      # the negacyclic mode, odd fold (halved)
    y = np.concatenate([ye + yo, ye - yo], axis=-1)
    assert oracle.rel_frobenius(y, oracle.cyclic_forward(x, W)) < 1e-12


def test_negacyclic_twiddle_table_is_cos_of_multiples_of_pi_over_8():
    import math
    src = open(os.path.join(ROOT, "group_wise_dft_b200", "csrc", "tc_transforms.cuh")).read()
    body = src[src.index("__host__ __device__ constexpr float cos_pi8(int m) {"):]
    body = body[:body.index("__host__ __device__ constexpr float sin_pi8")]
    consts = dict(re.findall(r"constexpr float (c\d) = ([0-9.]+)f;", body))
    vals = {}
    for case, expr in re.findall(r"case (\d+): return ([^;]+);", body):
        e = expr.strip().rstrip("f")
        sign = -1.0 if e.startswith("-") else 1.0
        e = e.lstrip("-")
        vals[int(case)] = sign * float(consts.get(e, e.rstrip("f")))
    vals[15] = float(consts["c1"])                               # the default case
    for m in range(16):
        assert abs(vals[m] - math.cos(m * math.pi / 8)) < 1e-7
        assert abs(vals[(m - 4) & 15] - math.sin(m * math.pi / 8)) < 1e-7   # sin_pi8(m) = cos_pi8(m - 4)


# ------------------------------------------------------------------ p4 (C_4) as super-fields


def c4_mma_list():
    """The C_4 MMA list in issue order, parsed from the kernel source."""
    src = _source()
    body = src[src.index("if (mode == kModeCyclic4) {\n    // Row r"):]
    body = body[: body.index("default:")]
    cases = re.findall(r"case (\d+): return \{([-\d, ]+)\};", body)
    return [tuple(int(v) for v in vals.split(",")) for _, vals in sorted(cases, key=lambda c: int(c[0]))]


C4_GROUP_COORD = [0, 2, 1, 3]   # TMEM groups [Re Y0, Im Y1, Re Y1, Re Y2] -> coordinate


def c4_panel_bytes(k, co):
    return 16 * co if k % 3 < 2 else 32 * co


def c4_panel_offset(k, co):
    return sum(c4_panel_bytes(i, co) for i in range(k))


def c4_entry(W, cout, o, cin, i):
    """C_4 block value: coordinates [Re0, Re1, Im1, Re2]; the 1/4 and the
    one-sided inverse's 2 folded in."""
    b = 0 if cout == 0 else (2 if cout == 3 else 1)
    m = np.arange(4)
    re = np.sum(W[o, i] * np.cos(2 * np.pi * m * b / 4)) / 4
    im = -np.sum(W[o, i] * np.sin(2 * np.pi * m * b / 4)) / 4
    if b != 1:
        return re
    out_re, in_re = cout == 1, cin == 1
    return 2 * ((re if in_re else -im) if out_re else (im if in_re else re))


def c4_pack(W, Fi4, Fo):
    """Fi4 C_4 input fields = Fi4 / 2 super-fields (the kernel's F_in)."""
    Fs = Fi4 // 2
    total = stage_offset(Fs, Fo, num_chunks(Fo) - 1, Fs // 16, 0)
    B = np.full(total // 2, np.nan)
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        for jp in range(Fs // 16):
            for hh in range(2):
                off = stage_offset(Fs, Fo, c, jp, hh) // 2
                for e in range(stage_bytes(co) // 2):
                    k = 0
                    while k + 1 < 6 and 2 * e >= c4_panel_offset(k + 1, co):
                        k += 1
                    w = e - c4_panel_offset(k, co) // 2
                    r, kind = divmod(k, 3)
                    if kind < 2:
                        kc, row, el = w // (hc * 8), (w // 8) % hc, w % 8
                        o, i = c * K_CO_MAX + hh * hc + row, 32 * jp + 16 * r + 2 * el + kc
                        cc = 0 if kind == 0 else 3
                        val = c4_entry(W, cc, o, cc, i)
                    else:
                        kc, row, el = w // (co * 8), (w // 8) % co, w % 8
                        o, i = c * K_CO_MAX + hh * hc + (row % hc), 32 * jp + 16 * r + 2 * el + kc
                        val = c4_entry(W, 2, o, 1, i) if row < hc else c4_entry(W, 1, o, 1, i)
                    assert np.isnan(B[off + e]), "two panel elements packed to one place"
                    B[off + e] = val
    assert not np.any(np.isnan(B)), "packed buffer has holes"
    return B


def c4_emulate(x, W):
    """x [T, Fi4, 4], W [Fo, Fi4, 4] -> y [T, Fo, 4] through the fused kernel's
    C_4 layout: the transform places coordinate q of a row's 16 C_4 fields in
    chunk pair q (even fields in chunk 2q, odd in 2q + 1), so the K index k of a
    K-step is field 2k (k < 8) or 2(k - 8) + 1 of the row."""
    T, Fi4, _ = x.shape
    Fo = W.shape[0]
    Fs = Fi4 // 2
    B = c4_pack(W, Fi4, Fo)
    X = np.fft.fft(x, axis=-1)
    Z = np.stack([X[..., 0].real, X[..., 1].real, X[..., 1].imag, X[..., 2].real], axis=-1)  # [T, Fi4, 4]
    kfield = np.array([2 * k if k < 8 else 2 * (k - 8) + 1 for k in range(16)])
    mmas = c4_mma_list()
    assert len(mmas) == 10
    acc_first = [any(m[3] >= e[3] and m[3] < e[3] + 1 + e[4] for e in mmas[:f]) for f, m in enumerate(mmas)]
    y = np.zeros((T, Fo, 4))
    for c in range(num_chunks(Fo)):
        co = chunk_fields(Fo, c)
        hc = co // 2
        D = [np.full((T, 4 * hc), np.nan) for _ in range(2)]
        for jp in range(Fs // 16):
            for f, (blk, pair, panel, dgroup, wide, neg, roff) in enumerate(mmas):
                A = Z[:, 32 * jp + 16 * blk + kfield, pair]          # [T, K = 16]: coordinate `pair`
                rows = co if wide else hc
                lbo = (c4_panel_bytes(panel, co) // 32) * 16
                for h in range(2):
                    start = stage_offset(Fs, Fo, c, jp, h) + c4_panel_offset(panel, co) + roff * hc * 16
                    n = np.arange(rows)[:, None]
                    k = np.arange(16)[None, :]
                    byte = start + (n // 8) * 128 + (n % 8) * 16 + (k // 8) * lbo + (k % 8) * 2
                    assert np.all(byte < stage_offset(Fs, Fo, c, jp, h) + stage_bytes(co))
                    prod = (A @ B[byte // 2].T) * (-1.0 if neg else 1.0)
                    cols = slice(dgroup * hc, dgroup * hc + rows)
                    if jp == 0 and not acc_first[f]:
                        D[h][:, cols] = prod
                    else:
                        D[h][:, cols] = D[h][:, cols] + prod
        g = np.arange(4)
        for h in range(2):
            assert not np.any(np.isnan(D[h])), "a TMEM column group was never written"
            Y = np.zeros((T, hc, 4))
            for kk in range(4):
                Y[:, :, C4_GROUP_COORD[kk]] = D[h][:, kk * hc:(kk + 1) * hc]
            yy = (Y[..., 0:1] + ((-1.0) ** g) * Y[..., 3:4] + Y[..., 1:2] * np.cos(np.pi * g / 2)
                  - Y[..., 2:3] * np.sin(np.pi * g / 2))
            y[:, c * K_CO_MAX + h * hc:c * K_CO_MAX + (h + 1) * hc, :] = yy
    return y


@pytest.mark.parametrize("Fi4,Fo", [(32, 32), (64, 96), (320, 64), (96, 160)])
def test_c4_tensor_core_layout_reproduces_the_layer(Fi4, Fo):
    rng = np.random.default_rng(Fi4 + Fo)
    x = rng.standard_normal((3, Fi4, 4))
    W = rng.standard_normal((Fo, Fi4, 4)) / np.sqrt(4 * Fi4)
    y = c4_emulate(x, W)
    ref = oracle.cyclic_forward(x, W)
    assert oracle.rel_frobenius(y, ref) < 1e-12



# ------------------------------------------------------------------ fp32 through split spectra


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("Cin,Cout", [(16, 32), (48, 64), (32, 160)])
def test_fp32_split_reaches_1e5_through_the_c8_layout(Cin, Cout):
    """fp32 C_8 on the bf16 MMAs: the pre-pass writes each field's spectrum (fp32)
    as [X_hi | X_lo | X_hi] (bf16; X_lo = bf16(X - X_hi)), the pack writes the
    weights as [W_hi | W_hi | W_lo] for those three blocks of Cin input fields,
    and one pass of the C_8 MMA list over the 3 Cin-wide layer sums
    X_hi W_hi + X_lo W_hi + X_hi W_lo.  With every rounding applied, the result
    must be within 1e-5 of the fp64 oracle (the fp32 tolerance)."""
    rng = np.random.default_rng(Cin + Cout)
    T = 5
    x = rng.standard_normal((T, Cin, 8)).astype(np.float32).astype(np.float64)
    W = (rng.standard_normal((Cout, Cin, 8)) / np.sqrt(8 * Cin)).astype(np.float32).astype(np.float64)
    X = x_coordinates(x).astype(np.float32).astype(np.float64)      # the pre-pass's fp32 spectra
    hi = _bf16(X)
    lo = _bf16(X - hi)
    Z = np.concatenate([hi, lo, hi], axis=1)

    def entry(cout, o, cin, i3):
        blk, i = divmod(i3, Cin)
        v = float(np.float32(spectrum_entry(W, cout, o, cin, i)))
        h = float(_bf16(v))
        return h if blk < 2 else float(_bf16(v - h))

    B = pack(W, 3 * Cin, Cout, entry=entry)
    y = emulate(None, W, Z=Z, B=B)
    err = oracle.rel_frobenius(y, oracle.cyclic_forward(x, W))
    assert err <= 1e-5, err
    # and the split is what gets there: hi parts alone stay at bf16 accuracy
    B_hi = pack(W, Cin, Cout, entry=lambda co_, o_, ci_, i_: float(_bf16(spectrum_entry(W, co_, o_, ci_, i_))))
    assert oracle.rel_frobenius(emulate(None, W, Z=hi, B=B_hi), oracle.cyclic_forward(x, W)) > 1e-4


@pytest.mark.parametrize("Cin,Cout", [(64, 32), (160, 64)])
def test_fp32_split_in_slices_reaches_1e5(Cin, Cout):
    """Wider fp32 layers run the split slice by slice: slice j takes input fields
    48 j .. 48 j + w - 1 (w <= 48, so its 3 w-wide layer fits the resident A
    operand) against its own packed [W_hi | W_hi | W_lo] panels, and the slices'
    fp32 outputs add up.  The sum must meet 1e-5 like the single-slice layer."""
    rng = np.random.default_rng(Cin + 7 * Cout)
    T = 4
    x = rng.standard_normal((T, Cin, 8)).astype(np.float32).astype(np.float64)
    W = (rng.standard_normal((Cout, Cin, 8)) / np.sqrt(8 * Cin)).astype(np.float32).astype(np.float64)
    X = x_coordinates(x).astype(np.float32).astype(np.float64)
    y = np.zeros((T, Cout, 8))
    for off in range(0, Cin, 48):
        w = min(48, Cin - off)
        Wj = W[:, off:off + w]
        hi = _bf16(X[:, off:off + w])
        lo = _bf16(X[:, off:off + w] - hi)

        def entry(cout, o, cin, i3, Wj=Wj, w=w):
            blk, i = divmod(i3, w)
            v = float(np.float32(spectrum_entry(Wj, cout, o, cin, i)))
            h = float(_bf16(v))
            return h if blk < 2 else float(_bf16(v - h))

        B = pack(Wj, 3 * w, Cout, entry=entry)
        y = (y + emulate(None, Wj, Z=np.concatenate([hi, lo, hi], axis=1), B=B)).astype(np.float32).astype(np.float64)
    err = oracle.rel_frobenius(y, oracle.cyclic_forward(x, W))
    assert err <= 1e-5, err
