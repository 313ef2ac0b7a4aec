"""The weight gradient without a caller workspace (eqlin_cyclic_weight_grad_noalloc).

Some callers of this library cannot allocate device memory (allocator or
memory-pool callbacks, frameworks that reserve all device memory up front,
plugins that must not touch the device heap); this entry point keeps its
partial sums in a fixed array inside the library instead.  The test calls it
through the raw C ABI twice in a row (the calls share that array) and checks
each result against eqlin_cyclic_weight_grad, which uses a workspace, and
against the fp64 oracle's weight gradient, within the tolerances of the other
GPU tests, and that a layer too large for the array is refused before
anything runs.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float(torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b))


@pytest.mark.parametrize("T,Cin,Cout,N,dtype", [
    (3000, 48, 80, 8, torch.bfloat16),
    (131072, 160, 160, 8, torch.bfloat16),
    (777, 16, 24, 5, torch.float32),
])
def test_noalloc_weight_grad_matches_workspace_version(T, Cin, Cout, N, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as eq
    import workloads as synth
    lib = eq.raw_lib()
    x, _, dy = synth.cyclic_backward_inputs(T, Cin, Cout, N, dtype, seed=T + Cin)
    x, dy = x.cuda(), dy.cuda()
    ref = eq.cyclic_weight_grad(x, dy)
    import oracle
    want = torch.from_numpy(oracle.cyclic_weight_grad(x.cpu().double().numpy(), dy.cpu().double().numpy()))
    code = eq.dtype_code(dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        dW = torch.full((Cout, Cin, N), -12288.0, dtype=dtype, device="cuda")
        rc = lib.eqlin_cyclic_weight_grad_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(dy.data_ptr()),
                                                  ctypes.c_void_p(dW.data_ptr()), T, N, Cin, Cout, code, stream)
        assert rc == eq.EQLIN_OK, lib.eqlin_last_error()
        torch.cuda.synchronize()
        err = _rel(dW, ref)
        assert err <= TOL[dtype], err
        err = _rel(dW.cpu(), want)
        assert err <= TOL[dtype], err
    assert eq.device_fault(reset=True) == 0


def test_noalloc_rejects_layers_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as eq
    lib = eq.raw_lib()
    p = ctypes.c_void_p(0x1000)   # never dereferenced: the call is refused before any launch
    # one token split of 1024 x 1024 fields at N = 16 is 64 MiB of fp32 partials
    rc = lib.eqlin_cyclic_weight_grad_noalloc(p, p, p, 64, 16, 1024, 1024, eq.EQLIN_BF16, None)
    assert rc == eq.EQLIN_ERR_SIZE
    assert b"scratch" in lib.eqlin_last_error()
