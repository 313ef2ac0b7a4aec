"""GPU parity of the Fourier-resident D8 layers (C ABI) against the fp64 oracle.

Features stay in the Fourier domain ([A1, A2, B1, B2, E00, E01, E10, E11]
per field) between layers, as in the Quick ViTs review (Key design 1); a
layer is the Schur block product (Key design 2), optionally followed by the
GELU round trip Q GELU(Q^T .); the MLP block is expand (with the round trip)
then contract.  Tolerances (relative Frobenius) as everywhere here: 1e-5 for
fp32 I/O, 2e-2 for bf16, 1e-3 for fp16; the MLP block's hidden features are
rounded to the I/O dtype between its two layers, which these bounds absorb.
Small cases compare every element, on CUDA cores and, for bf16 shapes it
takes (F_in % 16 == 0 up to 160, F_out % 32 == 0), on the fused tensor-core
kernel; the full-size block (T = 131072, 160 -> 640 -> 160 fields, bf16: the
expansion on tensor cores, the contraction on CUDA cores) compares sampled
token rows (the oracle is independent per token).  Equivariance: for every element u of D8 the block
commutes with u's action on Fourier coordinates, R_u = Q P_u Q^T per field.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2, torch.float16: 1e-3}


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _pack(eq, w):
    return eq.d8_fourier_pack_weights(*[b.cuda() for b in w])


LINEAR = [
    # T, F_in, F_out, dtype
    (64, 4, 16, torch.float32),
    (77, 20, 7, torch.float32),
    (1, 3, 5, torch.float32),
    (300, 16, 64, torch.bfloat16),
    (129, 40, 24, torch.float16),
    (50, 160, 640, torch.bfloat16),
]


def _paths(eq, F_in, F_out, dtype):
    """CUDA cores always; the fused tensor-core kernel where it takes the shape
    (wider than 160 input fields: in column slices, the binding providing the
    workspace)."""
    tc = dtype == torch.bfloat16 and F_in % 16 == 0 and F_in <= 8 * 160 and F_out % 32 == 0
    return [eq.PATH_SIMT] + ([eq.PATH_TC] if tc else [])


@pytest.mark.parametrize("T,F_in,F_out,dtype", LINEAR + [(129, 160, 64, torch.bfloat16),
                                                         (1, 32, 32, torch.bfloat16),
                                                         (100, 640, 160, torch.bfloat16),
                                                         (77, 176, 64, torch.bfloat16)])
@pytest.mark.parametrize("gelu", [False, True])
def test_fourier_linear_matches_the_oracle(eq, T, F_in, F_out, dtype, gelu):
    z, w1, _ = synth.d8_mlp_inputs(T, F_in, F_out, dtype, seed=T + F_in + F_out)
    pack = _pack(eq, w1)
    ref = oracle.d8_fourier_linear(_np(z), *[_np(b) for b in w1])
    if gelu:
        ref = oracle.d8_gelu_roundtrip(ref)
    for path in _paths(eq, F_in, F_out, dtype):
        y = eq.d8_fourier_linear(z.cuda(), pack, F_out, roundtrip_gelu=gelu, path=path)
        torch.cuda.synchronize()
        assert oracle.rel_frobenius(_np(y), ref) <= TOL[dtype], path
    assert eq.device_fault(reset=True) == 0


MLP = [(100, 8, 32, torch.float32), (333, 16, 64, torch.bfloat16), (64, 12, 48, torch.float16)]


@pytest.mark.parametrize("T,F,Fh,dtype", MLP)
def test_fourier_mlp_block_matches_the_oracle(eq, T, F, Fh, dtype):
    z, w1, w2 = synth.d8_mlp_inputs(T, F, Fh, dtype, seed=7 * T + F)
    y = eq.d8_fourier_mlp(z.cuda(), _pack(eq, w1), _pack(eq, w2), Fh)
    torch.cuda.synchronize()
    ref = oracle.d8_mlp_block(_np(z), [_np(b) for b in w1], [_np(b) for b in w2])
    assert oracle.rel_frobenius(_np(y), ref) <= TOL[dtype]


def test_fourier_mlp_block_is_equivariant(eq):
    T, F, Fh = 200, 8, 32
    z, w1, w2 = synth.d8_mlp_inputs(T, F, Fh, torch.float32, seed=17)
    p1, p2 = _pack(eq, w1), _pack(eq, w2)
    base = _np(eq.d8_fourier_mlp(z.cuda(), p1, p2, Fh))
    Q = oracle.d8_Q()
    for u in oracle.d8_elements():
        R = Q @ oracle.d8_regular_perm(u) @ Q.T
        zu = torch.from_numpy(np.einsum("cd,tid->tic", R, _np(z))).float()
        got = _np(eq.d8_fourier_mlp(zu.cuda(), p1, p2, Fh))
        want = np.einsum("cd,tid->tic", R, base)
        assert oracle.rel_frobenius(got, want) <= 1e-5, u


def test_full_size_block_sampled_rows(eq):
    T, F, Fh = 131072, 160, 640
    z, w1, w2 = synth.d8_mlp_inputs(T, F, Fh, torch.bfloat16, seed=4)
    y = eq.d8_fourier_mlp(z.cuda(), _pack(eq, w1), _pack(eq, w2), Fh)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(T, 64, replace=False))
    ref = oracle.d8_mlp_block(_np(z[rows]), [_np(b) for b in w1], [_np(b) for b in w2])
    assert oracle.rel_frobenius(_np(y)[rows], ref) <= TOL[torch.bfloat16]
    assert eq.device_fault(reset=True) == 0
