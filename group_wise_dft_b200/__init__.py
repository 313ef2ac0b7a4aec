"""Python binding of libeqlin (the C ABI in include/eqlin.h).

Argument marshalling only: every step of the layers runs in the library's
CUDA kernels.  torch supplies device memory and the current stream.  Importing
this package fails loudly if the shared library has not been built; there is
no CPU or PyTorch fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libeqlin.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python group_wise_dft_b200/build.py` "
        "(nvcc, sm_100a).  There is no fallback path.")

_lib = ctypes.CDLL(LIB_PATH)

EQLIN_OK = 0
EQLIN_ERR_INVALID_ARG = 1
EQLIN_ERR_UNSUPPORTED = 2
EQLIN_ERR_ALIGN = 3
EQLIN_ERR_CUDA = 4
EQLIN_ERR_SIZE = 5
EQLIN_F32 = 0
EQLIN_BF16 = 1
EQLIN_F16 = 2
PATH_AUTO = 0
PATH_SIMT = 1
PATH_TC = 2

_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t

_SIGS = {
    "eqlin_last_error": (ctypes.c_char_p, []),
    "eqlin_version": (_i, []),
    "eqlin_device_fault": (_i, [_i]),
    "eqlin_cyclic_spectrum_bytes": (_sz, [_i, _i, _i, _i]),
    "eqlin_cyclic_weight_spectrum": (_i, [_vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_cyclic_forward": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "eqlin_cyclic_forward_ex": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp]),
    "eqlin_cyclic_auto_path": (_i, [_i, _i, _i, _i]),
    "eqlin_cyclic_forward_workspace_bytes": (_sz, [_i64, _i, _i, _i, _i]),
    "eqlin_cyclic_forward_ws": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_cyclic_weight_spectrum_adjoint": (_i, [_vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_cyclic_backward_data": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "eqlin_cyclic_backward_data_ex": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp]),
    "eqlin_cyclic_weight_grad_workspace_bytes": (_sz, [_i64, _i, _i, _i, _i]),
    "eqlin_cyclic_weight_grad": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_cyclic_weight_grad_ex": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp, _sz, _i, _vp]),
    "eqlin_cyclic_weight_grad_noalloc": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "eqlin_d8_weight_bytes": (_sz, [_i, _i]),
    "eqlin_d8_pack_weights": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _sz, _vp]),
    "eqlin_d8_forward": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _vp]),
    "eqlin_d8_forward_ex": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "eqlin_d8_auto_path": (_i, [_i, _i]),
    "eqlin_d8_fourier_weight_bytes": (_sz, [_i, _i, _i]),
    "eqlin_d8_fourier_pack_weights": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_d8_fourier_linear": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _vp]),
    "eqlin_d8_fourier_linear_ex": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp]),
    "eqlin_d8_fourier_workspace_bytes": (_sz, [_i64, _i, _i, _i]),
    "eqlin_d8_fourier_linear_ws": (_i, [_vp, _vp, _vp, _i64, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_d8_fourier_mlp_workspace_bytes": (_sz, [_i64, _i, _i, _i]),
    "eqlin_d8_fourier_mlp_ws": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp, _sz, _vp]),
    "eqlin_d8_fourier_mlp": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _i, _i, _i, _vp]),
    "eqlin_selftest_wait_timeout": (_i, [ctypes.c_uint64, _i, _vp, _vp]),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class EqlinError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _lib.eqlin_last_error().decode(errors="replace")
        super().__init__(f"{where} failed with code {code}: {msg}")
        self.code = code


def _check(rc: int, where: str):
    if rc != EQLIN_OK:
        raise EqlinError(rc, where)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return EQLIN_F32
    if dt == torch.bfloat16:
        return EQLIN_BF16
    if dt == torch.float16:
        return EQLIN_F16
    raise TypeError(f"unsupported dtype {dt}")


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev_ptr(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def library_path() -> str:
    return LIB_PATH


def version() -> int:
    return _lib.eqlin_version()


def device_fault(reset: bool = True) -> int:
    return _lib.eqlin_device_fault(1 if reset else 0)


EQLIN_FAULT_SELFTEST = 0x1FF


def selftest_wait_timeout(limit_ns: int, arrive: bool = False, device=None) -> torch.Tensor:
    """Launch the bounded-wait self-test; returns a device int64 tensor that
    receives the wait's duration in ns (read it after a synchronize)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    elapsed = torch.zeros(1, dtype=torch.int64, device=device)
    rc = _lib.eqlin_selftest_wait_timeout(int(limit_ns), 1 if arrive else 0, _dev_ptr(elapsed, "elapsed"),
                                          _stream_ptr(device))
    _check(rc, "eqlin_selftest_wait_timeout")
    return elapsed


# ------------------------------------------------------------------ cyclic


def cyclic_spectrum_bytes(N: int, Cin: int, Cout: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_cyclic_spectrum_bytes(N, Cin, Cout, dtype_code(dtype)))


def cyclic_auto_path(N: int, Cin: int, Cout: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_cyclic_auto_path(N, Cin, Cout, dtype_code(dtype)))


def cyclic_weight_spectrum(W: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """W [Cout, Cin, N] (device) -> opaque spectrum buffer (uint8 device tensor)."""
    Cout, Cin, N = W.shape
    nbytes = cyclic_spectrum_bytes(N, Cin, Cout, W.dtype)
    if nbytes == 0:
        raise EqlinError(EQLIN_ERR_UNSUPPORTED, "eqlin_cyclic_spectrum_bytes")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    rc = _lib.eqlin_cyclic_weight_spectrum(_dev_ptr(W, "W"), N, Cin, Cout, dtype_code(W.dtype),
                                           _dev_ptr(out, "Wspec"), out.numel(), _stream_ptr(W.device))
    _check(rc, "eqlin_cyclic_weight_spectrum")
    return out


def cyclic_forward(x: torch.Tensor, Wspec: torch.Tensor, Cout: int, y: torch.Tensor | None = None,
                   path: int = PATH_AUTO) -> torch.Tensor:
    """x [T, Cin, N] (device) -> y [T, Cout, N] through the half spectrum."""
    T, Cin, N = x.shape
    if y is None:
        y = torch.empty((T, Cout, N), dtype=x.dtype, device=x.device)
    if tuple(y.shape) != (T, Cout, N) or y.dtype != x.dtype:
        raise ValueError("y has the wrong shape or dtype")
    rc = _lib.eqlin_cyclic_forward_ex(_dev_ptr(x, "x"), _dev_ptr(Wspec, "Wspec"), _dev_ptr(y, "y"),
                                      T, N, Cin, Cout, dtype_code(x.dtype), path,
                                      _stream_ptr(x.device))
    _check(rc, "eqlin_cyclic_forward")
    return y


def cyclic_forward_workspace_bytes(T: int, N: int, Cin: int, Cout: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_cyclic_forward_workspace_bytes(T, N, Cin, Cout, dtype_code(dtype)))


def cyclic_forward_ws(x: torch.Tensor, Wspec: torch.Tensor, Cout: int, y: torch.Tensor | None = None,
                      path: int = PATH_AUTO, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """x [T, Cin, N] (device) -> y [T, Cout, N]; with a workspace (a device byte
    tensor, allocated here when not given and needed), C_16 layers take the
    two-pass tensor-core path."""
    T, Cin, N = x.shape
    if y is None:
        y = torch.empty((T, Cout, N), dtype=x.dtype, device=x.device)
    if tuple(y.shape) != (T, Cout, N) or y.dtype != x.dtype:
        raise ValueError("y has the wrong shape or dtype")
    need = cyclic_forward_workspace_bytes(T, N, Cin, Cout, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    rc = _lib.eqlin_cyclic_forward_ws(_dev_ptr(x, "x"), _dev_ptr(Wspec, "Wspec"), _dev_ptr(y, "y"), T, N, Cin,
                                      Cout, dtype_code(x.dtype), path, _dev_ptr(workspace, "workspace"),
                                      workspace.numel(), _stream_ptr(x.device))
    _check(rc, "eqlin_cyclic_forward_ws")
    return y


def cyclic_weight_spectrum_adjoint(W: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """W [Cout, Cin, N] (device, the forward's weight) -> opaque spectrum of the
    backward data pass (the layer Cout -> Cin with the reflected, transposed weight)."""
    Cout, Cin, N = W.shape
    nbytes = cyclic_spectrum_bytes(N, Cout, Cin, W.dtype)
    if nbytes == 0:
        raise EqlinError(EQLIN_ERR_UNSUPPORTED, "eqlin_cyclic_spectrum_bytes")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    rc = _lib.eqlin_cyclic_weight_spectrum_adjoint(_dev_ptr(W, "W"), N, Cin, Cout, dtype_code(W.dtype),
                                                   _dev_ptr(out, "Wspec"), out.numel(),
                                                   _stream_ptr(W.device))
    _check(rc, "eqlin_cyclic_weight_spectrum_adjoint")
    return out


def cyclic_backward_data(dy: torch.Tensor, Wspec_adj: torch.Tensor, Cin: int,
                         dx: torch.Tensor | None = None, path: int = PATH_AUTO) -> torch.Tensor:
    """dy [T, Cout, N] (device) -> dx [T, Cin, N], with the spectrum from
    cyclic_weight_spectrum_adjoint."""
    T, Cout, N = dy.shape
    if dx is None:
        dx = torch.empty((T, Cin, N), dtype=dy.dtype, device=dy.device)
    if tuple(dx.shape) != (T, Cin, N) or dx.dtype != dy.dtype:
        raise ValueError("dx has the wrong shape or dtype")
    rc = _lib.eqlin_cyclic_backward_data_ex(_dev_ptr(dy, "dy"), _dev_ptr(Wspec_adj, "Wspec"),
                                            _dev_ptr(dx, "dx"), T, N, Cin, Cout, dtype_code(dy.dtype),
                                            path, _stream_ptr(dy.device))
    _check(rc, "eqlin_cyclic_backward_data")
    return dx


def cyclic_weight_grad_workspace_bytes(T: int, N: int, Cin: int, Cout: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, dtype_code(dtype)))


def cyclic_weight_grad(x: torch.Tensor, dy: torch.Tensor, dW: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, path: int = PATH_AUTO) -> torch.Tensor:
    """x [T, Cin, N], dy [T, Cout, N] (device) -> dW [Cout, Cin, N].  The
    workspace (a device byte tensor) is allocated here when not given.
    path: PATH_AUTO (tensor cores for N = 8, bf16), PATH_SIMT or PATH_TC."""
    T, Cin, N = x.shape
    Cout = dy.shape[1]
    if tuple(dy.shape) != (T, Cout, N) or dy.dtype != x.dtype:
        raise ValueError("dy has the wrong shape or dtype")
    if dW is None:
        dW = torch.empty((Cout, Cin, N), dtype=x.dtype, device=x.device)
    if tuple(dW.shape) != (Cout, Cin, N) or dW.dtype != x.dtype:
        raise ValueError("dW has the wrong shape or dtype")
    need = cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    rc = _lib.eqlin_cyclic_weight_grad_ex(_dev_ptr(x, "x"), _dev_ptr(dy, "dy"), _dev_ptr(dW, "dW"), T, N,
                                          Cin, Cout, dtype_code(x.dtype), _dev_ptr(workspace, "workspace"),
                                          workspace.numel(), path, _stream_ptr(x.device))
    _check(rc, "eqlin_cyclic_weight_grad_ex")
    return dW


# ------------------------------------------------------------------ D8


def d8_weight_bytes(C: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_d8_weight_bytes(C, dtype_code(dtype)))


def d8_auto_path(C: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_d8_auto_path(C, dtype_code(dtype)))


def d8_pack_weights(wA1, wA2, wB1, wB2, wE, out: torch.Tensor | None = None) -> torch.Tensor:
    F = wA1.shape[0]
    C = 8 * F
    nbytes = d8_weight_bytes(C, wA1.dtype)
    if nbytes == 0:
        raise EqlinError(EQLIN_ERR_UNSUPPORTED, "eqlin_d8_weight_bytes")
    for w, shp in ((wA1, (F, F)), (wA2, (F, F)), (wB1, (F, F)), (wB2, (F, F)), (wE, (2 * F, 2 * F))):
        if tuple(w.shape) != shp or w.dtype != wA1.dtype:
            raise ValueError("D8 weight blocks have inconsistent shapes or dtypes")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=wA1.device)
    rc = _lib.eqlin_d8_pack_weights(_dev_ptr(wA1, "wA1"), _dev_ptr(wA2, "wA2"), _dev_ptr(wB1, "wB1"),
                                    _dev_ptr(wB2, "wB2"), _dev_ptr(wE, "wE"), C, dtype_code(wA1.dtype),
                                    _dev_ptr(out, "Wpack"), out.numel(), _stream_ptr(wA1.device))
    _check(rc, "eqlin_d8_pack_weights")
    return out


def d8_forward(x: torch.Tensor, Wpack: torch.Tensor, fuse_gelu: bool = False,
               y: torch.Tensor | None = None, path: int = PATH_AUTO) -> torch.Tensor:
    """x [T, C/8, 8] (device) -> y [T, C/8, 8]."""
    T, F, eight = x.shape
    if eight != 8:
        raise ValueError("x must be [T, C/8, 8]")
    if y is None:
        y = torch.empty_like(x)
    if y.shape != x.shape or y.dtype != x.dtype:
        raise ValueError("y has the wrong shape or dtype")
    rc = _lib.eqlin_d8_forward_ex(_dev_ptr(x, "x"), _dev_ptr(Wpack, "Wpack"), _dev_ptr(y, "y"), T,
                                  8 * F, 1 if fuse_gelu else 0, dtype_code(x.dtype), path,
                                  _stream_ptr(x.device))
    _check(rc, "eqlin_d8_forward")
    return y


def d8_fourier_weight_bytes(F_in: int, F_out: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_d8_fourier_weight_bytes(F_in, F_out, dtype_code(dtype)))


def d8_fourier_pack_weights(wA1, wA2, wB1, wB2, wE, out: torch.Tensor | None = None) -> torch.Tensor:
    """Blocks of a Fourier-domain D8 layer F_in -> F_out: wA1..wB2 [F_out, F_in],
    wE [2 F_out, 2 F_in] (device) -> the opaque pack."""
    F_out, F_in = wA1.shape
    for w, shp in ((wA1, (F_out, F_in)), (wA2, (F_out, F_in)), (wB1, (F_out, F_in)), (wB2, (F_out, F_in)),
                   (wE, (2 * F_out, 2 * F_in))):
        if tuple(w.shape) != shp or w.dtype != wA1.dtype:
            raise ValueError("D8 weight blocks have inconsistent shapes or dtypes")
    nbytes = d8_fourier_weight_bytes(F_in, F_out, wA1.dtype)
    if nbytes == 0:
        raise EqlinError(EQLIN_ERR_UNSUPPORTED, "eqlin_d8_fourier_weight_bytes")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=wA1.device)
    rc = _lib.eqlin_d8_fourier_pack_weights(_dev_ptr(wA1, "wA1"), _dev_ptr(wA2, "wA2"), _dev_ptr(wB1, "wB1"),
                                            _dev_ptr(wB2, "wB2"), _dev_ptr(wE, "wE"), F_in, F_out,
                                            dtype_code(wA1.dtype), _dev_ptr(out, "Wpack"), out.numel(),
                                            _stream_ptr(wA1.device))
    _check(rc, "eqlin_d8_fourier_pack_weights")
    return out


def d8_fourier_linear(z: torch.Tensor, Wpack: torch.Tensor, F_out: int, roundtrip_gelu: bool = False,
                      y: torch.Tensor | None = None, path: int = PATH_AUTO) -> torch.Tensor:
    """z [T, F_in, 8] Fourier coordinates (device) -> y [T, F_out, 8]; with
    roundtrip_gelu, y = Q GELU(Q^T blocks(z))."""
    T, F_in, eight = z.shape
    if eight != 8:
        raise ValueError("z must be [T, F_in, 8]")
    if y is None:
        y = torch.empty((T, F_out, 8), dtype=z.dtype, device=z.device)
    if tuple(y.shape) != (T, F_out, 8) or y.dtype != z.dtype:
        raise ValueError("y has the wrong shape or dtype")
    need = int(_lib.eqlin_d8_fourier_workspace_bytes(T, F_in, F_out, dtype_code(z.dtype)))
    ws = torch.empty(need, dtype=torch.uint8, device=z.device) if need else None
    rc = _lib.eqlin_d8_fourier_linear_ws(_dev_ptr(z, "z"), _dev_ptr(Wpack, "Wpack"), _dev_ptr(y, "y"), T,
                                         F_in, F_out, 1 if roundtrip_gelu else 0, dtype_code(z.dtype), path,
                                         _dev_ptr(ws, "workspace") if ws is not None else None, need,
                                         _stream_ptr(z.device))
    _check(rc, "eqlin_d8_fourier_linear_ws")
    return y


def d8_fourier_mlp_workspace_bytes(T: int, F: int, F_hidden: int, dtype: torch.dtype) -> int:
    return int(_lib.eqlin_d8_fourier_mlp_workspace_bytes(T, F, F_hidden, dtype_code(dtype)))


def d8_fourier_mlp(z: torch.Tensor, W1pack: torch.Tensor, W2pack: torch.Tensor, F_hidden: int,
                   hidden: torch.Tensor | None = None, y: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The MLP block in the Fourier domain: z [T, F, 8] -> expand to F_hidden,
    GELU round trip, contract back to [T, F, 8].  workspace: a device byte
    tensor of d8_fourier_mlp_workspace_bytes (allocated here when not given);
    it lets a wide contraction run on tensor cores."""
    T, F, eight = z.shape
    if eight != 8:
        raise ValueError("z must be [T, F, 8]")
    if hidden is None:
        hidden = torch.empty((T, F_hidden, 8), dtype=z.dtype, device=z.device)
    if y is None:
        y = torch.empty_like(z)
    if tuple(hidden.shape) != (T, F_hidden, 8) or hidden.dtype != z.dtype:
        raise ValueError("hidden has the wrong shape or dtype")
    if y.shape != z.shape or y.dtype != z.dtype:
        raise ValueError("y has the wrong shape or dtype")
    need = d8_fourier_mlp_workspace_bytes(T, F, F_hidden, z.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=z.device)
    rc = _lib.eqlin_d8_fourier_mlp_ws(_dev_ptr(z, "z"), _dev_ptr(W1pack, "W1pack"), _dev_ptr(W2pack, "W2pack"),
                                      _dev_ptr(hidden, "hidden"), _dev_ptr(y, "y"), T, F, F_hidden,
                                      dtype_code(z.dtype),
                                      _dev_ptr(workspace, "workspace") if workspace is not None else None,
                                      workspace.numel() if workspace is not None else 0, _stream_ptr(z.device))
    _check(rc, "eqlin_d8_fourier_mlp_ws")
    return y


# ------------------------------------------------------------------ host-resident data


class HostPipeline:
    """A forward over host-resident (pinned) activations, in token chunks.

    The host->device copy of chunk i+1, the kernel on chunk i and the
    device->host copy of chunk i-1 run on three CUDA streams, so the two PCIe
    directions and the kernel overlap.  ``forward(x_dev, y_dev)`` is one of
    this module's forward calls bound to its weights; the two device staging
    buffers per direction are allocated here, once.  ``run`` is ordered after
    the work already queued on the current stream, and the current stream
    waits for its last copy, so events recorded around it time the whole job.
    """

    def __init__(self, forward, x_tail, y_tail, dtype, device, chunk_tokens: int = 16384):
        self.forward = forward
        self.chunk = int(chunk_tokens)
        self.xd = [torch.empty((self.chunk, *x_tail), dtype=dtype, device=device) for _ in range(2)]
        self.yd = [torch.empty((self.chunk, *y_tail), dtype=dtype, device=device) for _ in range(2)]
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(device) for _ in range(3))
        self.device = device

    def run(self, x_host: torch.Tensor, y_host: torch.Tensor) -> torch.Tensor:
        T = x_host.shape[0]
        if not (x_host.is_pinned() and y_host.is_pinned()):
            raise ValueError("host buffers must be pinned")
        cur = torch.cuda.current_stream(self.device)
        for s in (self.s_in, self.s_run, self.s_out):
            s.wait_stream(cur)
        n = (T + self.chunk - 1) // self.chunk
        ran = [None] * n
        out = [None] * n
        for i in range(n):
            b, t0 = i & 1, i * self.chunk
            t1 = min(T, t0 + self.chunk)
            xd, yd = self.xd[b][: t1 - t0], self.yd[b][: t1 - t0]
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(ran[i - 2])          # the kernel is done reading xd
                xd.copy_(x_host[t0:t1], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(self.s_in)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(landed)
                if i >= 2:
                    self.s_run.wait_event(out[i - 2])         # yd has been copied out
                self.forward(xd, yd)
                ran[i] = torch.cuda.Event()
                ran[i].record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ran[i])
                y_host[t0:t1].copy_(yd, non_blocking=True)
                out[i] = torch.cuda.Event()
                out[i].record(self.s_out)
        for s in (self.s_in, self.s_run, self.s_out):
            cur.wait_stream(s)
        return y_host


def raw_lib() -> ctypes.CDLL:
    """The loaded ctypes library (for tests of the raw C ABI)."""
    return _lib
