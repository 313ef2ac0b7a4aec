"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, plus equivariance of the GPU outputs.

Tolerances (relative Frobenius error against the oracle): 1e-5 for fp32 I/O,
2e-2 for bf16 I/O with fp32 accumulation.  Every case compares every element:
small cases at once, the full-size workloads and the multi-tile cases in
blocks of token rows with every 128-token tile held to the tolerance on its
own (tests/fullcheck.py).  Outputs start as NaN, so an unwritten row fails
both the oracle comparison and the equivariance checks.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth
from tests.fullcheck import GUARD, check_all_rows, check_guards, guarded

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


def _paths(eq, kind, *shape_args):
    paths = [eq.PATH_SIMT]
    if kind == "cyclic" and eq.cyclic_auto_path(*shape_args) == eq.PATH_TC:
        paths.append(eq.PATH_TC)
    if kind == "d8" and eq.d8_auto_path(*shape_args) == eq.PATH_TC:
        paths.append(eq.PATH_TC)
    return paths


_guarded = guarded
_check_guards = check_guards


def _multi_tile_T():
    """Tokens for three 128-token tiles per CTA pair of the tensor-core grid
    (one pair per two SMs) plus a ragged tail of 77."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return (sms // 2) * 128 * 3 + 77


def run_cyclic(eq, x, W, path):
    Cout, Cin, N = W.shape
    Ws = eq.cyclic_weight_spectrum(W)
    buf, y, pad = _guarded((x.shape[0], Cout, N), x.dtype)
    eq.cyclic_forward(x, Ws, Cout, y=y, path=path)
    torch.cuda.synchronize()
    _check_guards(buf, pad)
    return y


SMALL_CYCLIC = [
    # T, Cin, Cout, N, dtype
    (64, 16, 16, 4, torch.float32),
    (1, 3, 5, 8, torch.float32),
    (127, 7, 9, 16, torch.float32),
    (33, 5, 37, 3, torch.float32),
    (50, 17, 2, 1, torch.float32),
    (257, 12, 20, 6, torch.float32),
    (1000, 40, 24, 5, torch.bfloat16),
    (777, 64, 48, 8, torch.bfloat16),
    (300, 33, 65, 16, torch.bfloat16),
    (515, 160, 160, 8, torch.bfloat16),
    (129, 16, 16, 8, torch.bfloat16),
    (2000, 96, 128, 8, torch.bfloat16),
    (333, 160, 32, 8, torch.bfloat16),
    (64, 48, 80, 2, torch.bfloat16),
    (300, 48, 32, 8, torch.bfloat16),
    (200, 16, 96, 8, torch.bfloat16),
    (129, 112, 224, 8, torch.bfloat16),
    (1, 160, 160, 8, torch.bfloat16),
    (64, 32, 64, 8, torch.bfloat16),
    (65, 32, 64, 8, torch.bfloat16),
    (300, 32, 288, 8, torch.bfloat16),     # five output chunks (the last one narrow): the wide-layer instance
    (1, 48, 256, 8, torch.bfloat16),
]


@pytest.mark.parametrize("T,Cin,Cout,N,dtype", SMALL_CYCLIC)
def test_cyclic_small_all_elements(eq, T, Cin, Cout, N, dtype):
    x, W = synth.cyclic_inputs(T, Cin, Cout, N, dtype, seed=T + Cin + N)
    ref = oracle.cyclic_forward(_np(x), _np(W))
    for path in _paths(eq, "cyclic", N, Cin, Cout, dtype):
        y = run_cyclic(eq, x.cuda(), W.cuda(), path)
        err = oracle.rel_frobenius(_np(y), ref)
        assert err <= TOL[dtype], (path, err)
    assert eq.device_fault(reset=True) == 0


def test_cyclic_fp32_matches_pages_precision(eq):
    """fp32 SIMT path stays within a few 1e-7 of the fp64 result (the pages
    report ~1e-7 in FP32)."""
    w = synth.CYCLIC_WORKLOADS["c4_t64_16x16_f32"]
    x, W = synth.workload_inputs(w)
    y = run_cyclic(eq, x.cuda(), W.cuda(), eq.PATH_SIMT)
    err = oracle.rel_frobenius(_np(y), oracle.cyclic_forward(_np(x), _np(W)))
    assert err < 1e-6


def test_cyclic_empty_input_is_noop(eq):
    x = torch.empty((0, 16, 8), dtype=torch.bfloat16, device="cuda")
    W = torch.randn(16, 16, 8, device="cuda").to(torch.bfloat16)
    Ws = eq.cyclic_weight_spectrum(W)
    y = torch.empty((0, 16, 8), dtype=torch.bfloat16, device="cuda")
    eq.cyclic_forward(x, Ws, 16, y=y)
    torch.cuda.synchronize()


def _cyclic_every_row(eq, x, W, paths, tol, shifts=()):
    """Every row of each path's output against the oracle (in row blocks),
    then shift equivariance over the whole output."""
    xd, Wd = x.cuda(), W.cuda()
    outs = {path: run_cyclic(eq, xd, Wd, path) for path in paths}
    W64 = _np(W)
    check_all_rows(outs, lambda r0, r1: oracle.cyclic_forward(_np(x[r0:r1]), W64), x.shape[0], tol)
    for path, y in outs.items():
        # equivariance on the whole GPU output: roll x by s along g -> y rolls by s
        for s in shifts:
            ys = run_cyclic(eq, torch.roll(xd, s, dims=-1), Wd, path)
            e = oracle.rel_frobenius(_np(ys), _np(torch.roll(y, s, dims=-1)))
            assert e <= tol, (path, "shift", s, e)
            del ys
    del outs


@pytest.mark.parametrize("name", list(synth.CYCLIC_WORKLOADS))
def test_cyclic_workloads(eq, name):
    w = synth.CYCLIC_WORKLOADS[name]
    x, W = synth.workload_inputs(w)
    _cyclic_every_row(eq, x, W, _paths(eq, "cyclic", w.N, w.Cin, w.Cout, w.torch_dtype),
                      TOL[w.torch_dtype], shifts=(1, w.N // 2))
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("Cin,Cout", [(160, 160), (64, 96), (160, 32), (48, 224), (160, 416)])
def test_cyclic_several_tiles_per_cta_pair(eq, Cin, Cout):
    """Three tiles per CTA pair and a ragged tail: the persistent kernel's
    next-tile prefetch, A-buffer reuse and phase flips, on every element."""
    T = _multi_tile_T()
    x, W = synth.cyclic_inputs(T, Cin, Cout, 8, torch.bfloat16, seed=T + Cin + Cout)
    paths = [eq.PATH_TC] if eq.cyclic_auto_path(8, Cin, Cout, torch.bfloat16) == eq.PATH_TC else [eq.PATH_SIMT]
    _cyclic_every_row(eq, x, W, paths, TOL[torch.bfloat16], shifts=(3,))
    assert eq.device_fault(reset=True) == 0


# ------------------------------------------------------------------ D8


def run_d8(eq, x, ws, gelu, path):
    Wp = eq.d8_pack_weights(*ws)
    buf, y, pad = _guarded(tuple(x.shape), x.dtype)
    eq.d8_forward(x, Wp, fuse_gelu=gelu, y=y, path=path)
    torch.cuda.synchronize()
    _check_guards(buf, pad)
    return y


SMALL_D8 = [
    (64, 16, False, torch.float32),
    (31, 24, True, torch.float32),
    (129, 128, True, torch.bfloat16),
    (300, 256, False, torch.bfloat16),
    (1000, 1280, True, torch.bfloat16),
    (77, 8, True, torch.bfloat16),
    (1, 256, True, torch.bfloat16),
    (130, 512, False, torch.bfloat16),
    (250, 768, True, torch.bfloat16),
]


@pytest.mark.parametrize("T,C,gelu,dtype", SMALL_D8)
def test_d8_small_all_elements(eq, T, C, gelu, dtype):
    x, *ws = synth.d8_inputs(T, C, dtype, seed=C + T)
    ref = oracle.d8_forward(_np(x), *[_np(w) for w in ws], fuse_gelu=gelu)
    for path in _paths(eq, "d8", C, dtype):
        y = run_d8(eq, x.cuda(), [w.cuda() for w in ws], gelu, path)
        err = oracle.rel_frobenius(_np(y), ref)
        assert err <= TOL[dtype], (path, err)


def _d8_every_row(eq, x, ws, gelu, paths, tol, elements):
    xd = x.cuda()
    wd = [v.cuda() for v in ws]
    outs = {path: run_d8(eq, xd, wd, gelu, path) for path in paths}
    ws64 = [_np(v) for v in ws]
    check_all_rows(outs, lambda r0, r1: oracle.d8_forward(_np(x[r0:r1]), *ws64, fuse_gelu=gelu),
                   x.shape[0], tol)
    for path, y in outs.items():
        # equivariance: the regular-action permutations commute with the layer
        for u in elements:
            P = torch.as_tensor(oracle.d8_regular_perm(u), dtype=torch.float32, device="cuda")
            perm = P.argmax(dim=1)                      # (P x)[g] = x[perm[g]]
            yu = run_d8(eq, xd[..., perm].contiguous(), wd, gelu, path)
            e = oracle.rel_frobenius(_np(yu), _np(y[..., perm]))
            assert e <= tol, (path, u, e)
            del yu
    del outs


@pytest.mark.parametrize("name", list(synth.D8_WORKLOADS))
def test_d8_workloads(eq, name):
    w = synth.D8_WORKLOADS[name]
    x, *ws = synth.workload_inputs(w)
    _d8_every_row(eq, x, ws, w.fuse_gelu, _paths(eq, "d8", w.C, w.torch_dtype), TOL[w.torch_dtype],
                  oracle.d8_elements()[1:])
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("C,gelu", [(1280, True), (512, False)])
def test_d8_several_tiles_per_cta_pair(eq, C, gelu):
    T = _multi_tile_T()
    x, *ws = synth.d8_inputs(T, C, torch.bfloat16, seed=T + C)
    paths = [eq.PATH_TC] if eq.d8_auto_path(C, torch.bfloat16) == eq.PATH_TC else [eq.PATH_SIMT]
    _d8_every_row(eq, x, ws, gelu, paths, TOL[torch.bfloat16], oracle.d8_elements()[1:3])
    assert eq.device_fault(reset=True) == 0


@pytest.mark.parametrize("kind", ["cyclic", "d8"])
def test_host_pipeline_matches_device_call(eq, kind):
    # chunks of 384 tokens over T = 1000 (a ragged last chunk, both staging
    # buffers reused): the pipelined host path must reproduce the device call
    # exactly (same kernel on the same rows)
    T = 1000
    if kind == "cyclic":
        x, W = synth.cyclic_inputs(T, 64, 96, 8, torch.bfloat16, seed=21)
        Ws = eq.cyclic_weight_spectrum(W.cuda())
        fwd = lambda xx, yy: eq.cyclic_forward(xx, Ws, 96, y=yy)
        x_tail, y_tail = (64, 8), (96, 8)
    else:
        x, *ws = synth.d8_inputs(T, 512, torch.bfloat16, seed=22)
        Wp = eq.d8_pack_weights(*[w.cuda() for w in ws])
        fwd = lambda xx, yy: eq.d8_forward(xx, Wp, fuse_gelu=True, y=yy)
        x_tail = y_tail = (64, 8)
    ref = torch.empty((T, *y_tail), dtype=x.dtype, device="cuda")
    fwd(x.cuda(), ref)
    pipe = eq.HostPipeline(fwd, x_tail, y_tail, x.dtype, torch.device("cuda"), chunk_tokens=384)
    x_pin = x.pin_memory()
    y_pin = torch.full((T, *y_tail), -12288.0, dtype=x.dtype).pin_memory()
    pipe.run(x_pin, y_pin)
    torch.cuda.synchronize()
    assert torch.equal(y_pin, ref.cpu())
    assert eq.device_fault(reset=True) == 0
