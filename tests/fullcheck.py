"""Helpers of the GPU parity tests: guarded output buffers and a comparison of
every token row with the oracle.

The oracle computes token rows independently, so a full-size output is
compared in blocks of rows; within a block every 128-token tile (the tensor-
core kernel's unit of work) must meet the tolerance on its own, so one wrong
or skipped tile cannot hide behind the rest of the tensor.  Output buffers
start as NaN inside and a fixed pattern in 4 KiB guard bands on both sides: a
row the kernel never writes stays NaN and fails every comparison, and a write
outside y changes a guard.
"""

import numpy as np
import torch

import oracle

GUARD = -12288.0          # exactly representable in bf16, fp16 and fp32
TILE = 128


def guarded(shape, dtype, device="cuda"):
    """(buffer, y view, pad): y is NaN, the pad elements on each side GUARD."""
    n = int(np.prod(shape))
    pad = 4096 // torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((n + 2 * pad,), GUARD, dtype=dtype, device=device)
    buf[pad:pad + n] = float("nan")
    return buf, buf[pad:pad + n].view(*shape), pad


def check_guards(buf, pad):
    head = buf[:pad].float()
    tail = buf[-pad:].float()
    assert torch.all(head == GUARD) and torch.all(tail == GUARD), "write outside y"


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_all_rows(outputs, oracle_rows, T, tol, block=16384):
    """Compare every token row of each GPU output with the oracle.

    outputs: {label: device tensor [T, ...]}; oracle_rows(r0, r1) returns the
    oracle's float64 rows r0..r1-1.  Asserts that every 128-row tile of every
    output is within `tol` (relative Frobenius) of the oracle and returns the
    largest tile error and the whole-tensor error per label."""
    sq_err = {k: 0.0 for k in outputs}
    sq_ref = 0.0
    worst = {k: 0.0 for k in outputs}
    for r0 in range(0, T, block):
        r1 = min(T, r0 + block)
        ref = oracle_rows(r0, r1)
        sq_ref += float(np.sum(ref * ref))
        for k, y in outputs.items():
            got = to_np(y[r0:r1])
            assert np.isfinite(got).all(), (k, "unwritten or non-finite rows", r0, r1)
            for t0 in range(0, r1 - r0, TILE):
                e = oracle.rel_frobenius(got[t0:t0 + TILE], ref[t0:t0 + TILE])
                assert e <= tol, (k, "tile at token", r0 + t0, e)
                worst[k] = max(worst[k], e)
            d = got - ref
            sq_err[k] += float(np.sum(d * d))
    whole = {k: (sq_err[k] / sq_ref) ** 0.5 if sq_ref > 0 else sq_err[k] ** 0.5 for k in outputs}
    for k, e in whole.items():
        assert e <= tol, (k, "whole tensor", e)
    return worst, whole
