"""GPU parity of the tensor-core weight gradient (C_8, bf16) through the C ABI.

Each case runs the tensor-core path and the CUDA-core path on the same seeded
inputs and compares both with the fp64 oracle (relative Frobenius, 2e-2 for
bf16 I/O, as for every bf16 result here).  The workspace starts as all-ones
bytes (an fp32 NaN), so a partial sum the kernel failed to write poisons dW.
Shapes cover ragged field counts (not multiples of 8, 32, 64 or 128), ragged
token counts, one token, several tiles in both field directions and many
token splits; the full-size case compares the two paths on the 160 x 160,
T = 131072 layer (the CUDA-core path accumulates the spectra in fp32, so it
is an independent check at that size) and the oracle on sampled channel
pairs.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run(eq, x, dy, path):
    T, Cin, N = x.shape
    Cout = dy.shape[1]
    need = eq.cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, x.dtype)
    ws = torch.full((max(need, 16),), 0xFF, dtype=torch.uint8, device="cuda")
    dW = eq.cyclic_weight_grad(x, dy, workspace=ws, path=path)
    torch.cuda.synchronize()
    return dW


CASES = [
    # T, Cin, Cout
    (1, 8, 8),
    (31, 8, 13),
    (64, 16, 16),
    (100, 136, 40),
    (257, 64, 64),
    (1000, 200, 72),
    (2049, 160, 160),
    (4099, 96, 384),
    (20000, 24, 40),
]


@pytest.mark.parametrize("T,Cin,Cout", CASES)
def test_tensor_core_weight_gradient_matches_the_oracle(eq, T, Cin, Cout):
    x, _W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, 8, torch.bfloat16, seed=T + 3 * Cin + Cout)
    ref = oracle.cyclic_weight_grad(_np(x), _np(dy))
    tc = run(eq, x.cuda(), dy.cuda(), eq.PATH_TC)
    simt = run(eq, x.cuda(), dy.cuda(), eq.PATH_SIMT)
    assert torch.isfinite(tc.float()).all()
    e_tc = oracle.rel_frobenius(_np(tc), ref)
    e_simt = oracle.rel_frobenius(_np(simt), ref)
    assert e_tc <= TOL, ("tc", e_tc)
    assert e_simt <= TOL, ("simt", e_simt)
    assert eq.device_fault(reset=True) == 0


def test_auto_path_takes_the_tensor_cores_for_bf16_c8(eq):
    x, _W, dy = synth.cyclic_backward_inputs(3000, 48, 80, 8, torch.bfloat16, seed=7)
    a = run(eq, x.cuda(), dy.cuda(), eq.PATH_AUTO)
    b = run(eq, x.cuda(), dy.cuda(), eq.PATH_TC)
    assert torch.equal(a, b)


def test_tensor_core_weight_gradient_is_deterministic(eq):
    x, _W, dy = synth.cyclic_backward_inputs(9000, 160, 160, 8, torch.bfloat16, seed=11)
    a = run(eq, x.cuda(), dy.cuda(), eq.PATH_TC)
    b = run(eq, x.cuda(), dy.cuda(), eq.PATH_TC)
    assert torch.equal(a, b)


def test_tensor_core_path_refuses_other_shapes(eq):
    x = torch.zeros((64, 16, 8), dtype=torch.float32, device="cuda")
    dy = torch.zeros((64, 16, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError):
        run(eq, x, dy, eq.PATH_TC)
    x = torch.zeros((64, 16, 4), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((64, 16, 4), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        run(eq, x, dy, eq.PATH_TC)
    x = torch.zeros((64, 5, 8), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((64, 16, 8), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        run(eq, x, dy, eq.PATH_TC)


def test_full_size_160x160_paths_agree_and_match_sampled_pairs(eq):
    T, Cin, Cout = 131072, 160, 160
    x, _W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, 8, torch.bfloat16, seed=3)
    xc, dyc = x.cuda(), dy.cuda()
    tc = run(eq, xc, dyc, eq.PATH_TC)
    simt = run(eq, xc, dyc, eq.PATH_SIMT)
    assert oracle.rel_frobenius(_np(tc), _np(simt)) <= TOL
    g = np.random.default_rng(0)
    o_sub = np.sort(g.choice(Cout, 6, replace=False))
    i_sub = np.sort(g.choice(Cin, 6, replace=False))
    ref = oracle.cyclic_weight_grad(_np(x[:, i_sub]), _np(dy[:, o_sub]))
    got = _np(tc)[np.ix_(o_sub, i_sub)]
    assert oracle.rel_frobenius(got, ref) <= TOL
    assert eq.device_fault(reset=True) == 0
