"""p4 (C_4) exactness on the GPU.

The Flash EQ-Linear page's "Specialization for p4" notes that the N = 4
transform matrices hold only 0, +-1 and +-1/2.  The CUDA-core path takes that
literally: the weight spectrum's twiddles are exact at quarter turns and the
forward and inverse transforms of x, y, dy and dW are additions.  Every step of
the fp32 layer is then exact for small-integer inputs (all intermediate values
are dyadic and far below 2^24), so the GPU must reproduce the fp64 oracle bit
for bit: forward, backward data pass and weight gradient.  A twiddle that is
off by one rounding (cos(pi/2) evaluated as 6e-17) leaves a nonzero residue
where the exact result is 0, and fails here.
"""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _ints(shape, lo, hi, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, shape, generator=g).to(torch.float32)


CASES = [(64, 16, 16), (77, 24, 40), (1, 3, 5), (300, 33, 7)]


@pytest.mark.parametrize("T,Cin,Cout", CASES)
def test_p4_layer_is_exact_for_integer_inputs(eq, T, Cin, Cout):
    x = _ints((T, Cin, 4), -3, 3, seed=T)
    W = _ints((Cout, Cin, 4), -3, 3, seed=T + 1)
    dy = _ints((T, Cout, 4), -3, 3, seed=T + 2)
    xn, Wn, dyn = (t.numpy().astype(np.float64) for t in (x, W, dy))

    y = eq.cyclic_forward(x.cuda(), eq.cyclic_weight_spectrum(W.cuda()), Cout)
    dx = eq.cyclic_backward_data(dy.cuda(), eq.cyclic_weight_spectrum_adjoint(W.cuda()), Cin)
    dW = eq.cyclic_weight_grad(x.cuda(), dy.cuda())
    torch.cuda.synchronize()

    assert np.array_equal(y.cpu().numpy().astype(np.float64), oracle.cyclic_forward(xn, Wn))
    assert np.array_equal(dx.cpu().numpy().astype(np.float64), oracle.cyclic_backward_data(dyn, Wn))
    assert np.array_equal(dW.cpu().numpy().astype(np.float64), oracle.cyclic_weight_grad(xn, dyn))
    assert eq.device_fault(reset=True) == 0
