"""C ABI: the library loads without a GPU, exports every entry point that
include/*.h declares, and its host-side validation returns the documented codes
before any device work (these calls launch nothing)."""

import ctypes
import glob
import os
import re

import pytest

import group_wise_dft_b200 as eq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"EQLIN_API\s+[\w\s\*]+?\b(eqlin_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("eqlin_cyclic_weight_spectrum", "eqlin_cyclic_forward", "eqlin_d8_forward",
                 "eqlin_d8_pack_weights", "eqlin_cyclic_spectrum_bytes", "eqlin_d8_weight_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(eq.library_path())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    from group_wise_dft_b200 import _SIGS
    assert set(declared_functions()) <= set(_SIGS)


def test_version():
    assert eq.version() == 102


def test_spectrum_bytes():
    import torch
    assert eq.cyclic_spectrum_bytes(8, 160, 160, torch.bfloat16) > 0
    assert eq.cyclic_spectrum_bytes(0, 16, 16, torch.float32) == 0
    assert eq.cyclic_spectrum_bytes(17, 16, 16, torch.float32) == 0
    assert eq.cyclic_spectrum_bytes(4, 0, 16, torch.float32) == 0
    # SIMT section alone is Cin*N*Cout fp32 values
    assert eq.cyclic_spectrum_bytes(4, 16, 16, torch.float32) >= 16 * 4 * 16 * 4
    assert eq.d8_weight_bytes(1280, torch.bfloat16) >= 8 * 160 * 160 * 4
    assert eq.d8_weight_bytes(12, torch.bfloat16) == 0


L = eq.raw_lib()
P = ctypes.c_void_p(0x1000)         # aligned, never dereferenced: calls fail before launch
MIS = ctypes.c_void_p(0x1008)


@pytest.mark.parametrize("args,code", [
    ((P, P, P, 64, 0, 16, 16, 0, 0), eq.EQLIN_ERR_UNSUPPORTED),       # N = 0
    ((P, P, P, 64, 17, 16, 16, 0, 0), eq.EQLIN_ERR_UNSUPPORTED),      # N > 16
    ((P, P, P, 64, 4, 0, 16, 0, 0), eq.EQLIN_ERR_INVALID_ARG),        # Cin = 0
    ((P, P, P, 64, 4, 16, 16, 7, 0), eq.EQLIN_ERR_UNSUPPORTED),       # bad dtype
    ((P, P, P, -1, 4, 16, 16, 0, 0), eq.EQLIN_ERR_INVALID_ARG),       # T < 0
    ((None, P, P, 64, 4, 16, 16, 0, 0), eq.EQLIN_ERR_INVALID_ARG),    # null x
    ((P, None, P, 64, 4, 16, 16, 0, 0), eq.EQLIN_ERR_INVALID_ARG),    # null Wspec
    ((MIS, P, P, 64, 4, 16, 16, 0, 0), eq.EQLIN_ERR_ALIGN),           # misaligned x
    ((P, P, MIS, 64, 4, 16, 16, 0, 0), eq.EQLIN_ERR_ALIGN),           # misaligned y
    ((None, None, None, 0, 4, 16, 16, 0, 0), eq.EQLIN_OK),            # T = 0 is a no-op
])
def test_cyclic_forward_host_validation(args, code):
    assert L.eqlin_cyclic_forward(*args) == code
    if code != eq.EQLIN_OK:
        assert len(L.eqlin_last_error()) > 0


def test_cyclic_forced_tc_path_rejects_unsupported_shapes():
    # fp32 never takes the tensor-core path
    rc = L.eqlin_cyclic_forward_ex(P, P, P, 64, 4, 16, 16, eq.EQLIN_F32, eq.PATH_TC, None)
    assert rc == eq.EQLIN_ERR_UNSUPPORTED
    rc = L.eqlin_cyclic_forward_ex(P, P, P, 64, 4, 16, 16, eq.EQLIN_F32, 9, None)
    assert rc == eq.EQLIN_ERR_INVALID_ARG


def test_spectrum_host_validation():
    assert L.eqlin_cyclic_weight_spectrum(P, 8, 16, 16, 1, P, 16, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_cyclic_weight_spectrum(None, 8, 16, 16, 1, P, 1 << 30, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_weight_spectrum(MIS, 8, 16, 16, 1, P, 1 << 30, None) == eq.EQLIN_ERR_ALIGN


@pytest.mark.parametrize("args,code", [
    ((P, P, P, 64, 12, 0, 1, 0), eq.EQLIN_ERR_UNSUPPORTED),           # C % 8 != 0
    ((P, P, P, 64, 0, 0, 1, 0), eq.EQLIN_ERR_UNSUPPORTED),            # C = 0
    ((P, P, P, 64, 16, 2, 1, 0), eq.EQLIN_ERR_INVALID_ARG),           # bad gelu flag
    ((P, P, P, -5, 16, 0, 1, 0), eq.EQLIN_ERR_INVALID_ARG),           # T < 0
    ((P, None, P, 64, 16, 0, 1, 0), eq.EQLIN_ERR_INVALID_ARG),
    ((P, P, MIS, 64, 16, 0, 1, 0), eq.EQLIN_ERR_ALIGN),
    ((None, None, None, 0, 16, 1, 1, 0), eq.EQLIN_OK),
])
def test_d8_forward_host_validation(args, code):
    assert L.eqlin_d8_forward(*args) == code


def test_d8_pack_host_validation():
    assert L.eqlin_d8_pack_weights(P, P, P, P, P, 16, 1, P, 8, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_d8_pack_weights(P, P, None, P, P, 16, 1, P, 1 << 30, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_d8_pack_weights(P, P, P, P, MIS, 16, 1, P, 1 << 30, None) == eq.EQLIN_ERR_ALIGN


def test_auto_path_queries():
    assert L.eqlin_cyclic_auto_path(4, 16, 16, eq.EQLIN_F32) == eq.PATH_SIMT
    assert L.eqlin_cyclic_auto_path(0, 16, 16, eq.EQLIN_F32) == -1
    assert L.eqlin_d8_auto_path(12, eq.EQLIN_BF16) == -1


def test_forced_tc_path_needs_32_byte_aligned_y():
    # the tensor-core epilogue writes y in 32-byte pieces: a 16- but not
    # 32-byte aligned y is refused before anything is launched
    y16 = ctypes.c_void_p(P.value + 16)
    rc = L.eqlin_cyclic_forward_ex(P, P, y16, 256, 8, 160, 160, eq.EQLIN_BF16, eq.PATH_TC, None)
    assert rc == eq.EQLIN_ERR_ALIGN
    assert b"32-byte" in L.eqlin_last_error()
    rc = L.eqlin_d8_forward_ex(P, P, y16, 256, 1280, 1, eq.EQLIN_BF16, eq.PATH_TC, None)
    assert rc == eq.EQLIN_ERR_ALIGN


def test_backward_spectrum_host_validation():
    # the adjoint spectrum is sized for the layer Cout -> Cin
    need = L.eqlin_cyclic_spectrum_bytes(8, 32, 16, 1)
    assert L.eqlin_cyclic_weight_spectrum_adjoint(P, 8, 16, 32, 1, P, need - 1, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_cyclic_weight_spectrum_adjoint(None, 8, 16, 32, 1, P, need, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_weight_spectrum_adjoint(MIS, 8, 16, 32, 1, P, need, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_cyclic_weight_spectrum_adjoint(P, 0, 16, 32, 1, P, need, None) == eq.EQLIN_ERR_UNSUPPORTED


def test_backward_data_host_validation():
    assert L.eqlin_cyclic_backward_data(P, P, MIS, 64, 4, 16, 16, 0, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_cyclic_backward_data(None, P, P, 64, 4, 16, 16, 0, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_backward_data(None, None, None, 0, 4, 16, 16, 0, None) == eq.EQLIN_OK
    # fp32 never takes the tensor-core path
    assert L.eqlin_cyclic_backward_data_ex(P, P, P, 64, 4, 16, 16, 0, eq.PATH_TC, None) == \
        eq.EQLIN_ERR_UNSUPPORTED


def test_weight_grad_host_validation():
    ws = L.eqlin_cyclic_weight_grad_workspace_bytes(4096, 8, 64, 64, 1)
    assert ws > 0 and ws % (64 * 64 * 8 * 4) == 0
    assert L.eqlin_cyclic_weight_grad_workspace_bytes(0, 8, 64, 64, 1) == 0
    assert L.eqlin_cyclic_weight_grad_workspace_bytes(4096, 17, 64, 64, 1) == 0
    assert L.eqlin_cyclic_weight_grad(P, P, P, 4096, 8, 64, 64, 1, P, ws - 1, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_cyclic_weight_grad(P, P, P, 4096, 8, 64, 64, 1, None, ws, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_weight_grad(P, P, None, 4096, 8, 64, 64, 1, P, ws, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_weight_grad(MIS, P, P, 4096, 8, 64, 64, 1, P, ws, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_cyclic_weight_grad(P, P, P, 4096, 8, 64, 64, 1, MIS, ws, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_cyclic_weight_grad(P, P, P, -1, 8, 64, 64, 1, P, ws, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_cyclic_weight_grad(P, P, P, 4096, 0, 64, 64, 1, P, ws, None) == eq.EQLIN_ERR_UNSUPPORTED


def test_weight_grad_path_selection_host_validation():
    bf16 = eq.EQLIN_BF16
    ws = L.eqlin_cyclic_weight_grad_workspace_bytes(131072, 8, 160, 160, bf16)
    # covers the tensor-core split count as well as the CUDA-core one
    assert ws % (160 * 160 * 8 * 4) == 0 and ws >= L.eqlin_cyclic_weight_grad_workspace_bytes(131072, 8, 160, 160, 0)
    assert L.eqlin_cyclic_weight_grad_ex(P, P, P, 4096, 8, 64, 64, bf16, P, ws, 7, None) == eq.EQLIN_ERR_INVALID_ARG
    # the tensor-core path is C_8 and bf16 only
    for N, Cin, dt in [(8, 64, 0), (8, 64, eq.EQLIN_F16), (4, 64, bf16), (16, 64, bf16), (8, 7, bf16)]:
        w = L.eqlin_cyclic_weight_grad_workspace_bytes(4096, N, Cin, 64, dt)
        assert L.eqlin_cyclic_weight_grad_ex(P, P, P, 4096, N, Cin, 64, dt, P, w, eq.PATH_TC, None) == \
            eq.EQLIN_ERR_UNSUPPORTED


def test_d8_fourier_host_validation():
    bf16 = eq.EQLIN_BF16
    # fp32: the CUDA-core section alone; bf16 160 -> 640: plus the fused kernel's weight stages
    assert L.eqlin_d8_fourier_weight_bytes(160, 640, 0) == 8 * 160 * 640 * 4
    assert L.eqlin_d8_fourier_weight_bytes(160, 640, bf16) > 8 * 160 * 640 * 4
    assert L.eqlin_d8_fourier_weight_bytes(640, 160, bf16) > 8 * 160 * 640 * 4   # four column-slice sections
    assert L.eqlin_d8_fourier_linear_ex(P, P, P, 64, 160, 640, 0, bf16, 7, None) == eq.EQLIN_ERR_INVALID_ARG
    for F_in, F_out, dt in [(160, 640, 0), (200, 160, bf16), (24, 64, bf16), (32, 48, bf16)]:
        assert L.eqlin_d8_fourier_linear_ex(P, P, P, 64, F_in, F_out, 0, dt, eq.PATH_TC, None) == \
            eq.EQLIN_ERR_UNSUPPORTED
    assert L.eqlin_d8_fourier_weight_bytes(0, 640, bf16) == 0
    assert L.eqlin_d8_fourier_weight_bytes(16, 16, 3) == 0
    nb = L.eqlin_d8_fourier_weight_bytes(16, 24, bf16)
    assert L.eqlin_d8_fourier_pack_weights(P, P, P, P, P, 16, 24, bf16, P, nb - 1, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_d8_fourier_pack_weights(P, None, P, P, P, 16, 24, bf16, P, nb, None) == \
        eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_d8_fourier_pack_weights(P, P, P, P, MIS, 16, 24, bf16, P, nb, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_d8_fourier_linear(P, P, P, 64, 16, 24, 2, bf16, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_d8_fourier_linear(P, P, P, -1, 16, 24, 0, bf16, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_d8_fourier_linear(P, P, MIS, 64, 16, 24, 0, bf16, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_d8_fourier_linear(None, None, None, 0, 16, 24, 1, bf16, None) == eq.EQLIN_OK
    assert L.eqlin_d8_fourier_linear(P, P, P, 64, 0, 24, 0, bf16, None) == eq.EQLIN_ERR_UNSUPPORTED
    assert L.eqlin_d8_fourier_mlp(P, P, P, None, P, 64, 16, 64, bf16, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_d8_fourier_mlp(P, P, P, MIS, P, 64, 16, 64, bf16, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_d8_fourier_mlp(None, None, None, None, None, 0, 16, 64, bf16, None) == eq.EQLIN_OK


def test_d8_fourier_slices_host_validation():
    bf16 = eq.EQLIN_BF16
    T = 1000
    # 640 -> 160 (four column slices of 160) needs four bf16 partial outputs
    assert L.eqlin_d8_fourier_workspace_bytes(T, 640, 160, bf16) == 4 * T * 160 * 16
    assert L.eqlin_d8_fourier_workspace_bytes(T, 176, 64, bf16) == 2 * T * 64 * 16
    assert L.eqlin_d8_fourier_workspace_bytes(T, 160, 640, bf16) == 0        # one slice: none
    assert L.eqlin_d8_fourier_workspace_bytes(T, 640, 160, 0) == 0           # fp32: CUDA cores
    assert L.eqlin_d8_fourier_workspace_bytes(T, 200, 64, bf16) == 0         # 200 % 16 != 0
    assert L.eqlin_d8_fourier_mlp_workspace_bytes(T, 160, 640, bf16) == 4 * T * 160 * 16
    ws = 4 * T * 160 * 16
    assert L.eqlin_d8_fourier_linear_ws(P, P, P, T, 640, 160, 0, bf16, eq.PATH_TC, None, 0, None) == \
        eq.EQLIN_ERR_SIZE
    assert L.eqlin_d8_fourier_linear_ws(P, P, P, T, 640, 160, 0, bf16, eq.PATH_TC, P, ws - 1, None) == \
        eq.EQLIN_ERR_SIZE
    assert L.eqlin_d8_fourier_linear_ws(P, P, P, T, 640, 160, 0, bf16, eq.PATH_TC,
                                        ctypes.c_void_p(P.value + 16), ws, None) == eq.EQLIN_ERR_ALIGN
    assert L.eqlin_d8_fourier_linear_ws(P, P, P, T, 200, 64, 0, bf16, eq.PATH_TC, P, 1 << 30, None) == \
        eq.EQLIN_ERR_UNSUPPORTED
    assert L.eqlin_d8_fourier_mlp_ws(P, P, P, P, P, T, 160, 640, bf16, MIS, ws, None) == eq.EQLIN_ERR_ALIGN


def test_fp32_tensor_core_route_host_validation():
    f32 = 0
    T = 1000
    # split activations: 3 Cin bf16 "fields" per token, 256-byte rounded
    need = L.eqlin_cyclic_forward_workspace_bytes(T, 8, 32, 64, f32)
    assert need == ((T * 96 * 16 + 255) // 256) * 256
    # wider layers run in slices of <= 48 input fields: the split activations of
    # all slices, then one fp32 partial output [T][Cout][8] for the later slices
    assert L.eqlin_cyclic_forward_workspace_bytes(T, 8, 64, 64, f32) == \
        ((T * 192 * 16 + 255) // 256) * 256 + ((T * 64 * 32 + 255) // 256) * 256
    assert L.eqlin_cyclic_forward_workspace_bytes(T, 8, 40, 64, f32) == 0      # Cin % 16 != 0
    assert L.eqlin_cyclic_forward_workspace_bytes(T, 8, 64, 48, f32) == 0      # Cout % 32 != 0
    assert L.eqlin_cyclic_forward_workspace_bytes(T, 8, 32, 64, eq.EQLIN_BF16) == 0
    # the fp32 spectrum carries the split weight stages
    assert L.eqlin_cyclic_spectrum_bytes(8, 32, 64, f32) > 32 * 64 * 8 * 4
    assert L.eqlin_cyclic_forward_ws(P, P, P, T, 8, 32, 64, f32, eq.PATH_TC, None, 0, None) == eq.EQLIN_ERR_SIZE
    assert L.eqlin_cyclic_forward_ws(P, P, P, T, 8, 32, 64, f32, eq.PATH_TC, MIS, need, None) == eq.EQLIN_ERR_SIZE


def test_selftest_wait_timeout_host_validation():
    assert L.eqlin_selftest_wait_timeout(999, 0, None, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_selftest_wait_timeout(10_000_000_001, 0, None, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_selftest_wait_timeout(1_000_000, 2, None, None) == eq.EQLIN_ERR_INVALID_ARG
    assert L.eqlin_selftest_wait_timeout(1_000_000, 0, ctypes.c_void_p(P.value + 4), None) == \
        eq.EQLIN_ERR_ALIGN
    assert eq.EQLIN_FAULT_SELFTEST == 0x1FF


def test_fp16_is_a_supported_dtype_on_the_cuda_core_path():
    assert L.eqlin_cyclic_spectrum_bytes(8, 16, 16, eq.EQLIN_F16) > 0
    assert L.eqlin_cyclic_spectrum_bytes(8, 16, 16, 3) == 0
    assert L.eqlin_d8_weight_bytes(64, eq.EQLIN_F16) > 0
    # fp16 takes the tensor cores only when asked for (C_8 only); AUTO keeps it on CUDA cores
    assert L.eqlin_cyclic_auto_path(8, 160, 160, eq.EQLIN_F16) == eq.PATH_SIMT
    assert L.eqlin_d8_auto_path(1280, eq.EQLIN_F16) == eq.PATH_SIMT
    rc = L.eqlin_cyclic_forward_ex(P, P, P, 64, 4, 160, 160, eq.EQLIN_F16, eq.PATH_TC, None)
    assert rc == eq.EQLIN_ERR_UNSUPPORTED
    # the fp16 spectrum carries the fused kernel's weight stages, like bf16
    assert L.eqlin_cyclic_spectrum_bytes(8, 160, 160, eq.EQLIN_F16) == \
        L.eqlin_cyclic_spectrum_bytes(8, 160, 160, eq.EQLIN_BF16)
    import torch
    assert eq.dtype_code(torch.float16) == eq.EQLIN_F16


def test_c16_workspace_queries_and_validation():
    ws = L.eqlin_cyclic_forward_workspace_bytes(65536, 16, 96, 384, eq.EQLIN_BF16)
    # e and d (8 slots of bf16 per input field) and the even half's output ye
    assert ws >= 2 * 65536 * 96 * 16 + 65536 * 384 * 16
    assert L.eqlin_cyclic_forward_workspace_bytes(65536, 8, 96, 384, eq.EQLIN_BF16) == 0
    assert L.eqlin_cyclic_forward_workspace_bytes(65536, 16, 96, 384, eq.EQLIN_F32) == 0
    assert L.eqlin_cyclic_forward_workspace_bytes(65536, 16, 100, 384, eq.EQLIN_BF16) == 0
    # a forced tensor-core path without a sufficient workspace is refused before any launch
    rc = L.eqlin_cyclic_forward_ws(P, P, P, 64, 16, 96, 384, eq.EQLIN_BF16, eq.PATH_TC, P, 16, None)
    assert rc == eq.EQLIN_ERR_SIZE
    rc = L.eqlin_cyclic_forward_ws(P, P, P, 64, 16, 96, 384, eq.EQLIN_BF16, eq.PATH_TC, None, 1 << 40, None)
    assert rc == eq.EQLIN_ERR_SIZE
    rc = L.eqlin_cyclic_forward_ws(P, P, MIS, 64, 16, 96, 384, eq.EQLIN_BF16, eq.PATH_TC, P, 1 << 40, None)
    assert rc == eq.EQLIN_ERR_ALIGN
    # the spectrum of a C_16 bf16 layer carries both halves' packed weights
    assert L.eqlin_cyclic_spectrum_bytes(16, 96, 384, eq.EQLIN_BF16) > \
        L.eqlin_cyclic_spectrum_bytes(16, 96, 384, eq.EQLIN_F32)
