"""GPU parity of fp32 C_8 layers on the tensor cores through split spectra.

A pre-pass computes each field's spectrum in fp32 and writes it as three bf16
blocks [X_hi | X_lo | X_hi] (X_lo = bf16(X - X_hi)); the weight spectrum is
packed as [W_hi | W_hi | W_lo]; one pass of the fused kernel over the 3 Cin-wide
layer (coordinates placed, not transformed; fp32 output) sums
X_hi W_hi + X_lo W_hi + X_hi W_lo.  The dropped X_lo W_lo and the two
truncations are each about 2^-18 relative, so the result must meet the fp32
tolerance of this build, 1e-5 relative Frobenius against the fp64 oracle (the
CPU layout emulation of the same arithmetic gives 4.5e-6).  Asked for with
PATH_TC through the workspace-taking forward; any Cin that is a multiple of 16,
in slices of at most 48 input fields (a 3 w-wide layer must fit the resident
A operand) whose fp32 outputs add up in a fixed order.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

pytestmark = pytest.mark.gpu

TOL = 1e-5


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _np(t):
    return t.detach().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T,Cin,Cout", [(515, 16, 32), (129, 48, 64), (1, 32, 32), (2000, 32, 160), (777, 48, 96),
                                         (515, 64, 32), (300, 160, 64), (129, 96, 96), (1, 112, 32),
                                         (3000, 160, 160)])
def test_fp32_on_tensor_cores_meets_1e5(eq, T, Cin, Cout):
    x, W = synth.cyclic_inputs(T, Cin, Cout, 8, torch.float32, seed=T + Cin)
    xd, Wd = x.cuda(), W.cuda()
    y = eq.cyclic_forward_ws(xd, eq.cyclic_weight_spectrum(Wd), Cout, path=eq.PATH_TC)
    torch.cuda.synchronize()
    assert y.dtype == torch.float32
    err = oracle.rel_frobenius(_np(y), oracle.cyclic_forward(_np(x), _np(W)))
    assert err <= TOL, err
    assert eq.device_fault(reset=True) == 0


def test_auto_keeps_fp32_on_cuda_cores(eq):
    assert eq.cyclic_auto_path(8, 32, 64, torch.float32) == eq.PATH_SIMT
