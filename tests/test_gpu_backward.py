"""GPU parity of the backward pass (through the C ABI) against the fp64 oracle.

dx: the backward data pass (the forward kernels with the adjoint spectrum);
dW: the weight gradient (per-bin token reduction into the caller's workspace).
Tolerances as for the forward (relative Frobenius): 1e-5 for fp32 I/O, 2e-2
for bf16 I/O with fp32 accumulation.  Every case compares every element: the
full-size workloads compare every row of dx in blocks (each 128-token tile
within the tolerance) and every channel pair of dW, and check the adjoint and
directional-derivative identities against the GPU forward over the whole
tensors.  Outputs start as NaN, so an unwritten element fails.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth
from tests.fullcheck import check_all_rows, check_guards, guarded

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


_guarded = guarded          # NaN inside, a pattern in 4 KiB guard bands
_check_guards = check_guards


def run_dx(eq, dy, W, path):
    Cout, Cin, N = W.shape
    Wa = eq.cyclic_weight_spectrum_adjoint(W)
    buf, dx, pad = _guarded((dy.shape[0], Cin, N), dy.dtype)
    eq.cyclic_backward_data(dy, Wa, Cin, dx=dx, path=path)
    torch.cuda.synchronize()
    _check_guards(buf, pad)
    return dx


def run_dw(eq, x, dy):
    T, Cin, N = x.shape
    Cout = dy.shape[1]
    buf, dW, pad = _guarded((Cout, Cin, N), x.dtype)
    ws = torch.full((max(eq.cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, x.dtype), 16),),
                    0xAB, dtype=torch.uint8, device="cuda")     # stale contents must not matter
    eq.cyclic_weight_grad(x, dy, dW=dW, workspace=ws)
    torch.cuda.synchronize()
    _check_guards(buf, pad)
    return dW


def _ip_scale(u, v):
    """Typical size of <u, v> for unrelated u, v: |u| |v| / sqrt(n).  An error
    in either operator (a sign, a transposition) moves the inner product by
    about this much, the GPU's rounding by about tol times it."""
    n = u.numel()
    return float(torch.linalg.vector_norm(u.double()) * torch.linalg.vector_norm(v.double())) / n ** 0.5


def _dx_paths(eq, N, Cin, Cout, dtype):
    # the backward data pass is the layer Cout -> Cin
    paths = [eq.PATH_SIMT]
    if eq.cyclic_auto_path(N, Cout, Cin, dtype) == eq.PATH_TC:
        paths.append(eq.PATH_TC)
    return paths


SMALL = [
    # T, Cin, Cout, N, dtype
    (64, 16, 16, 4, torch.float32),
    (1, 3, 5, 8, torch.float32),
    (127, 7, 9, 16, torch.float32),
    (33, 5, 37, 3, torch.float32),
    (50, 17, 2, 1, torch.float32),
    (600, 40, 33, 5, torch.float32),
    (1000, 40, 24, 5, torch.bfloat16),
    (777, 64, 48, 8, torch.bfloat16),
    (300, 33, 65, 16, torch.bfloat16),
    (515, 160, 160, 8, torch.bfloat16),
    (333, 32, 160, 8, torch.bfloat16),
    (129, 64, 96, 8, torch.bfloat16),
]


@pytest.mark.parametrize("T,Cin,Cout,N,dtype", SMALL)
def test_backward_data_small_all_elements(eq, T, Cin, Cout, N, dtype):
    x, W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, N, dtype, seed=T + Cout + N)
    ref = oracle.cyclic_backward_data(_np(dy), _np(W))
    for path in _dx_paths(eq, N, Cin, Cout, dtype):
        dx = run_dx(eq, dy.cuda(), W.cuda(), path)
        err = oracle.rel_frobenius(_np(dx), ref)
        assert err <= TOL[dtype], (path, err)
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("T,Cin,Cout,N,dtype", SMALL)
def test_weight_grad_small_all_elements(eq, T, Cin, Cout, N, dtype):
    x, W, dy = synth.cyclic_backward_inputs(T, Cin, Cout, N, dtype, seed=T + Cin + 2 * N)
    ref = oracle.cyclic_weight_grad(_np(x), _np(dy))
    dW = run_dw(eq, x.cuda(), dy.cuda())
    err = oracle.rel_frobenius(_np(dW), ref)
    assert err <= TOL[dtype], err
    assert eq.device_fault(reset=True) == 0


def test_weight_grad_is_deterministic(eq):
    x, W, dy = synth.cyclic_backward_inputs(5000, 48, 80, 8, torch.bfloat16, seed=31)
    a = run_dw(eq, x.cuda(), dy.cuda())
    b = run_dw(eq, x.cuda(), dy.cuda())
    assert torch.equal(a, b)


def test_weight_grad_of_no_tokens_is_zero(eq):
    x = torch.empty((0, 16, 8), dtype=torch.float32, device="cuda")
    dy = torch.empty((0, 24, 8), dtype=torch.float32, device="cuda")
    dW = run_dw(eq, x, dy)
    assert torch.all(dW == 0)


def test_backward_data_of_no_tokens_is_noop(eq):
    W = torch.randn(16, 16, 8, device="cuda").to(torch.bfloat16)
    Wa = eq.cyclic_weight_spectrum_adjoint(W)
    dy = torch.empty((0, 16, 8), dtype=torch.bfloat16, device="cuda")
    eq.cyclic_backward_data(dy, Wa, 16)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", list(synth.CYCLIC_WORKLOADS))
def test_backward_workloads(eq, name):
    w = synth.CYCLIC_WORKLOADS[name]
    x, W, dy = synth.cyclic_backward_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, w.seed + 100)
    tol = TOL[w.torch_dtype]
    xd, Wd, dyd = x.cuda(), W.cuda(), dy.cuda()
    Ws = eq.cyclic_weight_spectrum(Wd)
    # dx: every row against the oracle (each 128-token tile within the
    # tolerance), the shift equivariance and the adjoint identity
    # <dx, u> = <dy, f(u; W)> over the whole tensors
    W64 = _np(W)
    dxs_by_path = {path: run_dx(eq, dyd, Wd, path) for path in _dx_paths(eq, w.N, w.Cin, w.Cout, w.torch_dtype)}
    check_all_rows(dxs_by_path, lambda r0, r1: oracle.cyclic_backward_data(_np(dy[r0:r1]), W64), w.T, tol)
    for path, dx in dxs_by_path.items():
        dxs = run_dx(eq, torch.roll(dyd, 1, dims=-1), Wd, path)
        e = oracle.rel_frobenius(_np(dxs), _np(torch.roll(dx, 1, dims=-1)))
        assert e <= tol, (name, path, "shift", e)
        del dxs
    fx = eq.cyclic_forward(xd, Ws, w.Cout)
    a = float(torch.sum(dx.double() * xd.double()))
    b = float(torch.sum(dyd.double() * fx.double()))
    assert abs(a - b) <= tol * _ip_scale(dx, xd), (a, b)
    del dx, fx
    # dW: every channel pair against the oracle, and <dW, V> = <dy, f(x; V)>
    dW = run_dw(eq, xd, dyd)
    ref = oracle.cyclic_weight_grad(_np(x), _np(dy))
    got = _np(dW)
    assert np.isfinite(got).all()
    err = oracle.rel_frobenius(got, ref)
    assert err <= tol, (name, "dW", err)
    for o in range(w.Cout):   # each output field's gradient on its own
        e = oracle.rel_frobenius(got[o], ref[o])
        assert e <= tol, (name, "dW row", o, e)
    V = torch.randn(w.Cout, w.Cin, w.N, device="cuda").to(w.torch_dtype)
    fv = eq.cyclic_forward(xd, eq.cyclic_weight_spectrum(V), w.Cout)
    a = float(torch.sum(dW.double() * V.double()))
    b = float(torch.sum(dyd.double() * fv.double()))
    assert abs(a - b) <= tol * _ip_scale(dW, V), (a, b)
    assert eq.device_fault(reset=True) == 0
