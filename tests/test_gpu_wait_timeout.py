"""Failure detection without a GPU fault: a bounded wait runs out and reports.

Every wait inside this library's kernels (on an mbarrier, a TMA completion or
the other CTA of a pair) is bounded: after its limit the kernel records a code
in a device fault word, stops issuing work and returns normally, and the host
reads the code with eqlin_device_fault.  These tests make one such wait run
out on purpose, with the same wait routine, in a one-warp diagnostic kernel
whose barrier nothing completes; no kernel traps, faults or hangs.  They
check that the code arrives, that the wait lasted about its limit, that the
first code recorded is kept, that a completed wait records nothing, that the
context still runs a layer correctly afterwards, and that a fault left in the
word does not stop later launches (each launch has its own fault epoch).
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_wise_dft_b200 as m
    assert m.device_fault(reset=True) == 0
    return m


def _layer_still_right(eq):
    x, W = synth.cyclic_inputs(300, 16, 24, 8, torch.float32, seed=9)
    y = eq.cyclic_forward(x.cuda(), eq.cyclic_weight_spectrum(W.cuda()), 24)
    torch.cuda.synchronize()
    ref = oracle.cyclic_forward(x.numpy().astype(np.float64), W.numpy().astype(np.float64))
    return oracle.rel_frobenius(y.cpu().numpy().astype(np.float64), ref) <= 1e-5


def test_a_wait_that_nothing_completes_gives_up_and_reports(eq):
    limit = 2_000_000   # 2 ms
    el = eq.selftest_wait_timeout(limit)
    torch.cuda.synchronize()
    assert eq.device_fault(reset=True) == eq.EQLIN_FAULT_SELFTEST
    ns = int(el.item())
    assert limit <= ns < limit + 50_000_000, ns
    assert _layer_still_right(eq)
    assert eq.device_fault(reset=True) == 0


def test_the_first_code_recorded_is_kept(eq):
    eq.selftest_wait_timeout(1_000_000)
    torch.cuda.synchronize()
    # a second launch's wait runs out too: the word keeps the first code
    el = eq.selftest_wait_timeout(3_000_000)
    torch.cuda.synchronize()
    assert 3_000_000 <= int(el.item()) < 100_000_000
    assert eq.device_fault(reset=True) == eq.EQLIN_FAULT_SELFTEST
    assert eq.device_fault(reset=True) == 0


def test_a_stale_fault_does_not_stop_later_launches(eq):
    """Without clearing the word, a later launch's waits still run to their
    ends: each launch gives up early only on a fault of its own."""
    eq.selftest_wait_timeout(1_000_000)
    torch.cuda.synchronize()
    # a completed wait of a later launch returns at once, as on a clean device
    el = eq.selftest_wait_timeout(1_000_000_000, arrive=True)
    torch.cuda.synchronize()
    assert int(el.item()) < 1_000_000
    # the tensor-core kernel (whose producer, issuer, transform and epilogue
    # warps wait on one another for microseconds at a time) still computes the
    # whole layer; before per-launch epochs it gave up once a wait passed 20 us
    T, F = 4 * 128 * 148 + 77, 160
    x, W = synth.cyclic_inputs(T, F, F, 8, torch.bfloat16, seed=21)
    y = torch.full((T, F, 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    eq.cyclic_forward(x.cuda(), eq.cyclic_weight_spectrum(W.cuda()), F, y=y, path=eq.PATH_TC)
    torch.cuda.synchronize()
    rows = synth.sample_rows(T, 512, 21)
    ref = oracle.cyclic_forward(x[rows].double().numpy(), W.double().numpy())
    got = y[torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    assert oracle.rel_frobenius(got, ref) <= 2e-2
    assert torch.isfinite(y).all()   # every row written
    assert eq.device_fault(reset=True) == eq.EQLIN_FAULT_SELFTEST
    assert eq.device_fault(reset=True) == 0


def test_a_completed_wait_returns_at_once_and_records_nothing(eq):
    el = eq.selftest_wait_timeout(1_000_000_000, arrive=True)
    torch.cuda.synchronize()
    assert eq.device_fault(reset=True) == 0
    assert int(el.item()) < 1_000_000
