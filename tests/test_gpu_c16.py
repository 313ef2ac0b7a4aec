"""GPU parity of the C_16 two-pass tensor-core path (eqlin_cyclic_forward_ws)
against the fp64 oracle, through the C ABI: the even half on the C_8 kernel,
the odd half on its negacyclic mode, joined in the caller's workspace.
Tolerance as for every bf16 path: relative Frobenius error <= 2e-2."""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth
from tests.fullcheck import GUARD, check_all_rows

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


def _run(eq, x, W, path, workspace=None):
    Cout, Cin, N = W.shape
    Ws = eq.cyclic_weight_spectrum(W)
    n = x.shape[0] * Cout * N
    pad = 2048
    buf = torch.full((n + 2 * pad,), GUARD, dtype=x.dtype, device="cuda")
    buf[pad:pad + n] = float("nan")   # an unwritten element stays NaN and fails every check
    y = buf[pad:pad + n].view(x.shape[0], Cout, N)
    eq.cyclic_forward_ws(x, Ws, Cout, y=y, path=path, workspace=workspace)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad].float() == GUARD) and torch.all(buf[-pad:].float() == GUARD), "write outside y"
    return y


@pytest.mark.parametrize("T,Cin,Cout", [(129, 16, 32), (515, 96, 384), (1, 160, 64), (300, 48, 96),
                                        (2000, 32, 32)])
def test_c16_tensor_core_path_small(eq, T, Cin, Cout):
    x, W = synth.cyclic_inputs(T, Cin, Cout, 16, torch.bfloat16, seed=T + Cin)
    ref = oracle.cyclic_forward(_np(x), _np(W))
    y = _run(eq, x.cuda(), W.cuda(), eq.PATH_TC)
    assert oracle.rel_frobenius(_np(y), ref) <= TOL
    assert eq.device_fault(reset=True) == 0


def test_c16_workload(eq):
    """Every row of the full C_16 workload (65536 tokens, 96 -> 384 fields)
    against the oracle, each 128-token tile within the tolerance, then shift
    equivariance over the whole output (NaN-filled y: unwritten rows fail)."""
    w = synth.CYCLIC_WORKLOADS["c16_t65536_96x384_bf16"]
    x, W = synth.workload_inputs(w)
    xd, Wd = x.cuda(), W.cuda()
    y = _run(eq, xd, Wd, eq.PATH_TC)
    W64 = _np(W)
    check_all_rows({"tc": y}, lambda r0, r1: oracle.cyclic_forward(_np(x[r0:r1]), W64), w.T, TOL)
    for s in (1, 8):
        ys = _run(eq, torch.roll(xd, s, dims=-1), Wd, eq.PATH_TC)
        assert oracle.rel_frobenius(_np(ys), _np(torch.roll(y, s, dims=-1))) <= TOL, s
        del ys
    assert eq.device_fault(reset=True) == 0


def test_c16_several_tiles_per_cta_pair(eq):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T = (sms // 2) * 128 * 3 + 77
    x, W = synth.cyclic_inputs(T, 96, 128, 16, torch.bfloat16, seed=T)
    y = _run(eq, x.cuda(), W.cuda(), eq.PATH_TC)
    W64 = _np(W)
    check_all_rows({"tc": y}, lambda r0, r1: oracle.cyclic_forward(_np(x[r0:r1]), W64), T, TOL)
    assert eq.device_fault(reset=True) == 0


def test_c16_auto_without_workspace_takes_the_cuda_core_path(eq):
    x, W = synth.cyclic_inputs(100, 32, 64, 16, torch.bfloat16, seed=5)
    Ws = eq.cyclic_weight_spectrum(W.cuda())
    tiny = torch.empty(256, dtype=torch.uint8, device="cuda")
    a = eq.cyclic_forward_ws(x.cuda(), Ws, 64, workspace=tiny)          # AUTO, workspace too small
    b = eq.cyclic_forward(x.cuda(), Ws, 64, path=eq.PATH_SIMT)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
