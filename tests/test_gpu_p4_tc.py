"""GPU parity of p4 (C_4, bf16) on the fused tensor-core kernel.

Pairs of C_4 fields ride the kernel's 8-slot geometry as super-fields: the
transform (additions only) places coordinate q of a row's 16 C_4 fields in
chunk pair q, 10 MMAs per K-slice cover bins 0, 2 (real) and 1 (complex), and
the epilogue inverts two fields per super-field.  Asked for with PATH_TC (AUTO
keeps C_4 on CUDA cores until this file passes).  Forward and backward data
pass against the fp64 oracle, relative Frobenius 2e-2 as for every bf16 result;
shapes cover one block pair (32 fields), the 320-field maximum, several output
chunks, a ragged token count and one token.
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


@pytest.mark.parametrize("T,Cin,Cout", [(515, 64, 64), (129, 320, 96), (1, 32, 32), (2000, 96, 160),
                                        (333, 32, 320)])
def test_p4_on_tensor_cores(eq, T, Cin, Cout):
    x, W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, 4, torch.bfloat16, seed=T + Cin + Cout)
    xd, Wd, dyd = x.cuda(), W.cuda(), dy.cuda()
    y = eq.cyclic_forward(xd, eq.cyclic_weight_spectrum(Wd), Cout, path=eq.PATH_TC)
    torch.cuda.synchronize()
    assert oracle.rel_frobenius(_np(y), oracle.cyclic_forward(_np(x), _np(W))) <= TOL
    if Cout % 32 == 0 and Cout <= 320 and Cin % 32 == 0:
        dx = eq.cyclic_backward_data(dyd, eq.cyclic_weight_spectrum_adjoint(Wd), Cin, path=eq.PATH_TC)
        torch.cuda.synchronize()
        assert oracle.rel_frobenius(_np(dx), oracle.cyclic_backward_data(_np(dy), _np(W))) <= TOL
    assert eq.device_fault(reset=True) == 0


def test_auto_keeps_p4_on_cuda_cores(eq):
    assert eq.cyclic_auto_path(4, 64, 64, torch.bfloat16) == eq.PATH_SIMT
