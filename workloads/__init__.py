"""Seeded synthetic inputs shared by the tests, the smoke run and the bench.

This module holds no arithmetic of the layers: it only draws random inputs
(torch CPU generator, float64 normals, then a cast to the I/O dtype) and names
the workloads.  Both the CUDA path and the fp64 oracle receive the same cast
values, so a comparison measures only the error of the path under test.

Recipe: ``torch.Generator().manual_seed(seed)``; draw x first, then the
weights in the order listed; weights are N(0, 1/(Cin*N)) for the cyclic layer
and N(0, 1/C) for the D8 layer.  Shapes follow ViT token batches (32 x 16x16 and
512 x 256 tokens) at ViT-H width 1280 and a 4x MLP expansion.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class CyclicWorkload:
    name: str
    T: int
    Cin: int
    Cout: int
    N: int
    dtype: str          # "f32" or "bf16"
    seed: int

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class D8Workload:
    name: str
    T: int
    C: int
    fuse_gelu: bool
    dtype: str
    seed: int

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


CYCLIC_WORKLOADS = {
    "c4_t64_16x16_f32": CyclicWorkload("c4_t64_16x16_f32", 64, 16, 16, 4, "f32", 0),
    "c8_t8192_64x64_bf16": CyclicWorkload("c8_t8192_64x64_bf16", 8192, 64, 64, 8, "bf16", 1),
    "c16_t65536_96x384_bf16": CyclicWorkload("c16_t65536_96x384_bf16", 65536, 96, 384, 16, "bf16", 2),
    "c8_t131072_160x160_bf16": CyclicWorkload("c8_t131072_160x160_bf16", 131072, 160, 160, 8, "bf16", 3),
    "c8_t131072_160x640_bf16": CyclicWorkload("c8_t131072_160x640_bf16", 131072, 160, 640, 8, "bf16", 3),
    # p4 at the same 1280 dense dimensions (320 C_4 fields), for the p4 tensor-core option
    "c4_t131072_320x320_bf16": CyclicWorkload("c4_t131072_320x320_bf16", 131072, 320, 320, 4, "bf16", 6),
}

D8_WORKLOADS = {
    "d8_t131072_c1280_gelu_bf16": D8Workload("d8_t131072_c1280_gelu_bf16", 131072, 1280, True, "bf16", 4),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def cyclic_inputs(T: int, Cin: int, Cout: int, N: int, dtype, seed: int):
    """x [T, Cin, N] ~ N(0, 1); W [Cout, Cin, N] ~ N(0, 1/(Cin*N)); cast to dtype."""
    g = _gen(seed)
    x = torch.randn(T, Cin, N, dtype=torch.float64, generator=g)
    W = torch.randn(Cout, Cin, N, dtype=torch.float64, generator=g) / math.sqrt(Cin * N)
    return x.to(dtype), W.to(dtype)


def cyclic_backward_inputs(T: int, Cin: int, Cout: int, N: int, dtype, seed: int):
    """x and W as cyclic_inputs(seed), then dy [T, Cout, N] ~ N(0, 1) from the same
    generator; cast to dtype."""
    g = _gen(seed)
    x = torch.randn(T, Cin, N, dtype=torch.float64, generator=g)
    W = torch.randn(Cout, Cin, N, dtype=torch.float64, generator=g) / math.sqrt(Cin * N)
    dy = torch.randn(T, Cout, N, dtype=torch.float64, generator=g)
    return x.to(dtype), W.to(dtype), dy.to(dtype)


def d8_inputs(T: int, C: int, dtype, seed: int):
    """x [T, C/8, 8] ~ N(0,1); wA1, wA2, wB1, wB2 [C/8, C/8] and wE [C/4, C/4] ~ N(0, 1/C)."""
    if C % 8:
        raise ValueError("C must be a multiple of 8")
    F = C // 8
    g = _gen(seed)
    x = torch.randn(T, F, 8, dtype=torch.float64, generator=g)
    s = 1.0 / math.sqrt(C)
    blocks = [torch.randn(F, F, dtype=torch.float64, generator=g) * s for _ in range(4)]
    wE = torch.randn(2 * F, 2 * F, dtype=torch.float64, generator=g) * s
    return (x.to(dtype), *[b.to(dtype) for b in blocks], wE.to(dtype))


def d8_mlp_inputs(T: int, F: int, F_hidden: int, dtype, seed: int):
    """Fourier-domain D8 MLP block: z [T, F, 8] ~ N(0, 1); the expansion's blocks
    (wA1, wA2, wB1, wB2 [F_hidden, F], wE [2 F_hidden, 2 F]) ~ N(0, 1/(8F)) and
    the contraction's ([F, F_hidden], [2F, 2 F_hidden]) ~ N(0, 1/(8 F_hidden)),
    i.e. N(0, 1/C_in) with C_in the layer's regular-representation width."""
    g = _gen(seed)
    z = torch.randn(T, F, 8, dtype=torch.float64, generator=g)

    def blocks(fo, fi):
        s = 1.0 / math.sqrt(8 * fi)
        ws = [torch.randn(fo, fi, dtype=torch.float64, generator=g) * s for _ in range(4)]
        ws.append(torch.randn(2 * fo, 2 * fi, dtype=torch.float64, generator=g) * s)
        return tuple(w.to(dtype) for w in ws)

    w1 = blocks(F_hidden, F)
    w2 = blocks(F, F_hidden)
    return z.to(dtype), w1, w2


def workload_inputs(w):
    if isinstance(w, CyclicWorkload):
        return cyclic_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, w.seed)
    return d8_inputs(w.T, w.C, w.torch_dtype, w.seed)


def sample_rows(T: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct token indices for sampled parity, always including the
    first and last token so both ends of the grid are covered."""
    count = min(count, T)
    rng = np.random.default_rng(seed + 1000003)
    rows = rng.choice(T, size=count, replace=False)
    rows[0] = 0
    if count > 1:
        rows[1] = T - 1
    return np.unique(rows)
