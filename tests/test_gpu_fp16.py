"""GPU parity for fp16 I/O (fp32 accumulation; CUDA cores, and for the C_8
layer also the fused tensor-core kernel) against the fp64 oracle on the same
fp16-rounded inputs.

The tolerance is derived from the arithmetic: the only rounding that the
oracle does not share is the final rounding of each output to fp16 (unit
roundoff 2^-11, a uniform error of RMS 2^-11 / sqrt(3) = 2.8e-4 relative) plus
fp32 accumulation (below 1e-6 here), so the relative Frobenius error must stay
under 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

pytestmark = pytest.mark.gpu

TOL_F16 = 1e-3


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T,Cin,Cout,N", [(300, 33, 65, 16), (515, 160, 160, 8), (1000, 40, 24, 5),
                                          (64, 16, 16, 4), (77, 9, 13, 1)])
def test_cyclic_fp16(eq, T, Cin, Cout, N):
    x, W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, N, torch.float16, seed=T + N)
    xd, Wd, dyd = x.cuda(), W.cuda(), dy.cuda()
    assert eq.cyclic_auto_path(N, Cin, Cout, torch.float16) == eq.PATH_SIMT
    y = eq.cyclic_forward(xd, eq.cyclic_weight_spectrum(Wd), Cout)
    dx = eq.cyclic_backward_data(dyd, eq.cyclic_weight_spectrum_adjoint(Wd), Cin)
    dW = eq.cyclic_weight_grad(xd, dyd)
    torch.cuda.synchronize()
    assert y.dtype == dx.dtype == dW.dtype == torch.float16
    assert oracle.rel_frobenius(_np(y), oracle.cyclic_forward(_np(x), _np(W))) <= TOL_F16
    assert oracle.rel_frobenius(_np(dx), oracle.cyclic_backward_data(_np(dy), _np(W))) <= TOL_F16
    assert oracle.rel_frobenius(_np(dW), oracle.cyclic_weight_grad(_np(x), _np(dy))) <= TOL_F16
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("T,Cin,Cout", [(515, 160, 160), (129, 64, 96), (1, 16, 32), (2000, 96, 128)])
def test_cyclic_fp16_on_tensor_cores(eq, T, Cin, Cout):
    """fp16 I/O on the fused kernel (asked for with PATH_TC; AUTO keeps fp16 on
    CUDA cores).  Its MMA operands are fp16 too: the spectra of x and the
    weight spectrum each add a rounding of unit 2^-11 per operand, about
    sqrt(2/3) 2^-11 = 4e-4 relative on the products, which with the output's
    2.8e-4 stays under the same 1e-3."""
    x, W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, 8, torch.float16, seed=T + Cin)
    xd, Wd, dyd = x.cuda(), W.cuda(), dy.cuda()
    y = eq.cyclic_forward(xd, eq.cyclic_weight_spectrum(Wd), Cout, path=eq.PATH_TC)
    # dx is the layer Cout -> Cin: on the tensor cores only when Cin is a multiple of 32 as well
    dx_path = eq.PATH_TC if Cin % 32 == 0 else eq.PATH_AUTO
    dx = eq.cyclic_backward_data(dyd, eq.cyclic_weight_spectrum_adjoint(Wd), Cin, path=dx_path)
    torch.cuda.synchronize()
    assert y.dtype == dx.dtype == torch.float16
    assert oracle.rel_frobenius(_np(y), oracle.cyclic_forward(_np(x), _np(W))) <= TOL_F16
    assert oracle.rel_frobenius(_np(dx), oracle.cyclic_backward_data(_np(dy), _np(W))) <= TOL_F16
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("T,C,gelu", [(129, 128, True), (300, 1280, True), (77, 8, False)])
def test_d8_fp16(eq, T, C, gelu):
    x, *ws = synth.d8_inputs(T, C, torch.float16, seed=C + T)
    Wp = eq.d8_pack_weights(*[w.cuda() for w in ws])
    y = eq.d8_forward(x.cuda(), Wp, fuse_gelu=gelu)
    torch.cuda.synchronize()
    ref = oracle.d8_forward(_np(x), *[_np(w) for w in ws], fuse_gelu=gelu)
    assert oracle.rel_frobenius(_np(y), ref) <= TOL_F16
