/*
 * eqlin.h -- C ABI of the B200 equivariant linear layers.
 *
 * Two layers, both mapping a batch of T tokens in the regular representation
 * of a finite group to another such batch:
 *
 *  1. Cyclic EQ-Linear over C_N ("Flash EQ-Linear: Accelerating Equivariant
 *     Linear Layers via Group-wise Discrete Fourier Transform",
 *     gist.science/paper/2607.21271, Technical Summary > Methodology):
 *
 *        y[t, o, g] = sum_i sum_h W[o, i, (g - h) mod N] * x[t, i, h]
 *
 *     computed exactly through the group-wise real DFT (Algorithmic Approach:
 *     convolution theorem, only the N/2+1 bins left by conjugate symmetry),
 *     a per-bin complex product over channels, and the inverse DFT.  The
 *     dense (Cout*N) x (Cin*N) matrix is never formed.
 *
 *  2. D8 Fourier-domain linear layer ("Quick ViTs: Speeding up Vision
 *     Transformers through Equivariance", papernotes.org ECCV2026 review,
 *     Key design 1 and 2): an 8x8 change of basis per field to the irreps
 *     A1, A2, B1, B2, E, four (C/8)-square products, one (C/4)-square product
 *     shared by E's two row coordinates, the change of basis back, and an
 *     optional GELU in the regular domain.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named x, y, W*, Wspec, Wpack are CUDA DEVICE memory owned by the
 *    caller.  The library never allocates, frees or retains them, and never
 *    synchronises the stream; all work is enqueued on `stream` (0 = legacy
 *    default stream).  Buffers must not overlap.
 *  - Activation layout: row-major, group slot fastest:
 *        x[T][Cin][N], y[T][Cout][N]     (cyclic)
 *        x[T][C/8][8], y[T][C/8][8]      (D8; slot j = r^j, slot 4+j = r^j s)
 *    so a token is a contiguous row of Cin*N (resp. C) values.
 *  - Weight matrices are [out][in] (the F.linear convention, y = W v).
 *  - dtype: EQLIN_F32 (fp32 in, fp32 out), EQLIN_BF16 (bf16 in/out, fp32
 *    accumulation) or EQLIN_F16 (fp16 in/out, fp32 accumulation; CUDA-core
 *    path only).  The same dtype applies to x, y and the weights.
 *  - x, y, W*, Wspec and Wpack must be 16-byte aligned.
 *  - No bias: the pages define none (an equivariant bias would have to be
 *    constant along the group axis; add it outside if needed).
 *  - Return value: EQLIN_OK or an EQLIN_ERR_* code.  Argument, shape and
 *    alignment errors are detected on the host before anything is launched;
 *    eqlin_last_error() then returns a message (per calling thread).
 *    EQLIN_ERR_CUDA reports a failed launch (cudaGetLastError).
 *  - Device kernels never trap.  A kernel whose bounded internal wait runs out
 *    records a code that eqlin_device_fault() returns.
 */
#ifndef EQLIN_H_
#define EQLIN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EQLIN_API __attribute__((visibility("default")))
#else
#define EQLIN_API
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA header. */
typedef struct CUstream_st *eqlin_stream_t;

enum {
  EQLIN_OK = 0,
  EQLIN_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad flag      */
  EQLIN_ERR_UNSUPPORTED = 2, /* shape or dtype outside the supported set   */
  EQLIN_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned           */
  EQLIN_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed       */
  EQLIN_ERR_SIZE = 5         /* a caller buffer is smaller than required   */
};

enum { EQLIN_F32 = 0, EQLIN_BF16 = 1, EQLIN_F16 = 2 };

/* Kernel selection for the *_ex entry points. */
enum {
  EQLIN_PATH_AUTO = 0,  /* library picks: tensor-core path where supported */
  EQLIN_PATH_SIMT = 1,  /* CUDA-core path: every supported shape and dtype  */
  EQLIN_PATH_TC = 2     /* tcgen05 tensor-core path (bf16, see below)       */
};

/* Message for the last error returned on this thread ("" if none). */
EQLIN_API const char *eqlin_last_error(void);

/* ABI version (major*100 + minor): 102. */
EQLIN_API int eqlin_version(void);

/* Fault word written by device code whose bounded wait ran out (0 = none).
 * Synchronises the device.  reset != 0 clears it afterwards.
 * The word keeps the FIRST code recorded since the last reset.  A launch whose
 * wait runs out stops only itself (its outputs are invalid): every launch has
 * its own fault epoch, and its waits give up early only when another wait of
 * the same launch gave up, so launches after a fault run normally whether or
 * not the word has been cleared.  A nonzero value therefore says that some
 * launch since the last reset failed, not that the latest one did. */
EQLIN_API int eqlin_device_fault(int reset);

/* Self-test of the bounded wait that every kernel's internal waits use (a
 * diagnostic; the pages have no counterpart).  Launches one warp on `stream`
 * that waits on a device barrier: with arrive = 0 nothing ever completes it,
 * so the wait gives up after limit_ns nanoseconds, records
 * EQLIN_FAULT_SELFTEST in the fault word (unless another code is already
 * there) and the kernel returns normally; with arrive = 1 the warp completes
 * the barrier itself first and the wait returns at once, recording nothing.
 * elapsed_ns: device pointer to one unsigned 64-bit value that receives the
 * wait's duration, or NULL.  limit_ns must be in 1000 .. 10^10 (10 s).
 * Asynchronous; read the result with eqlin_device_fault. */
#define EQLIN_FAULT_SELFTEST 0x1ff
EQLIN_API int eqlin_selftest_wait_timeout(uint64_t limit_ns, int arrive, void *elapsed_ns,
                                          eqlin_stream_t stream);

/* ---------------------------------------------------------------- cyclic */

/* Bytes of the weight-spectrum buffer for (N, Cin, Cout, dtype).
 * Supported: 1 <= N <= 16, Cin >= 1, Cout >= 1, dtype EQLIN_F32/EQLIN_BF16/EQLIN_F16.
 * Returns 0 for unsupported arguments. */
EQLIN_API size_t eqlin_cyclic_spectrum_bytes(int N, int Cin, int Cout, int dtype);

/* Weight spectrum (Flash EQ-Linear, Algorithmic Approach: frequency-domain
 * transformation of the group-circulant weight):
 *     What[k, o, i] = (1/N) sum_m W[o, i, m] exp(-2 pi i m k / N),
 *     k = 0 .. floor(N/2)   (the bins left by conjugate symmetry).
 * W: device [Cout][Cin][N] of `dtype`.  Wspec: device buffer of at least
 * eqlin_cyclic_spectrum_bytes(...) bytes, written with an opaque layout that
 * eqlin_cyclic_forward reads back for the same (N, Cin, Cout, dtype).  The
 * 1/N of the inverse transform is folded in here.  Run once per weight. */
EQLIN_API int eqlin_cyclic_weight_spectrum(const void *W, int N, int Cin, int Cout, int dtype,
                                 void *Wspec, size_t Wspec_bytes, eqlin_stream_t stream);

/* Forward pass y = EQ-Linear(x) through the half spectrum.
 * x: device [T][Cin][N], y: device [T][Cout][N], both `dtype`.
 * Wspec: written by eqlin_cyclic_weight_spectrum with the same arguments.
 * T = 0 is a no-op.  Supported: as for the spectrum; the tensor-core path
 * additionally needs dtype EQLIN_BF16, N == 8, Cin % 16 == 0,
 * 16 <= Cin <= 160, Cout % 32 == 0 (AUTO falls back to SIMT otherwise; TC
 * returns EQLIN_ERR_UNSUPPORTED), and y 32-byte aligned (AUTO falls back to
 * SIMT otherwise; TC returns EQLIN_ERR_ALIGN). */
EQLIN_API int eqlin_cyclic_forward(const void *x, const void *Wspec, void *y, int64_t T, int N,
                         int Cin, int Cout, int dtype, eqlin_stream_t stream);
EQLIN_API int eqlin_cyclic_forward_ex(const void *x, const void *Wspec, void *y, int64_t T, int N,
                            int Cin, int Cout, int dtype, int path, eqlin_stream_t stream);

/* Which path EQLIN_PATH_AUTO takes for these arguments (EQLIN_PATH_SIMT or
 * EQLIN_PATH_TC), or -1 if unsupported. */
EQLIN_API int eqlin_cyclic_auto_path(int N, int Cin, int Cout, int dtype);

/* Forward pass with a caller workspace.  For N = 16, bf16, 16 <= Cin <= 160
 * with Cin % 16 == 0 and Cout % 32 == 0, the layer runs on the tensor-core
 * kernel in two passes: it splits exactly into a C_8 cyclic layer on
 * e_h = x_h + x_{h+8} and a C_8 negacyclic layer (the product modulo z^8 + 1)
 * on d_h = x_h - x_{h+8}, with y_g = Y_e,g + Y_o,g and y_{g+8} = Y_e,g - Y_o,g
 * (the 1/2 of each is in the weight spectrum).  e, d and the even half's
 * output live in `workspace` (the odd half's epilogue reads that output and
 * writes y itself): caller-owned device memory, 256-byte aligned, of at least
 * eqlin_cyclic_forward_workspace_bytes(T, N, Cin, Cout, dtype) bytes (0 when no
 * such path applies).  For N = 8, fp32, Cin % 16 == 0 and Cout % 32 == 0,
 * EQLIN_PATH_TC runs the layer on the tensor cores at fp32 accuracy (1e-5):
 * a pre-pass writes each field's fp32 spectrum as bf16 X_hi and
 * X_lo = bf16(X - X_hi) into the workspace, and each slice of at most 48
 * input fields is one pass of the fused kernel summing X_hi W_hi + X_lo W_hi
 * + X_hi W_lo; the slices' fp32 outputs add up in a fixed order (the later
 * slices' partial output also lives in the workspace).  AUTO keeps fp32 on
 * the CUDA cores.  Every other case, or AUTO with a missing or short
 * workspace, is eqlin_cyclic_forward_ex; a forced EQLIN_PATH_TC without a
 * sufficient workspace returns EQLIN_ERR_SIZE. */
EQLIN_API size_t eqlin_cyclic_forward_workspace_bytes(int64_t T, int N, int Cin, int Cout, int dtype);
EQLIN_API int eqlin_cyclic_forward_ws(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                            int Cout, int dtype, int path, void *workspace, size_t workspace_bytes,
                            eqlin_stream_t stream);

/* ------------------------------------------------------- cyclic backward */

/* Backward data pass: for y = EQ-Linear(x; W), the gradient of sum(dy * y)
 * with respect to x is
 *     dx[t, i, h] = sum_o sum_g W[o, i, (g - h) mod N] dy[t, o, g],
 * which is the same layer applied to dy (Cout -> Cin) with the reflected,
 * transposed weight V[i, o, m] = W[o, i, (-m) mod N]; its spectrum is the
 * conjugate transpose of W's (Flash EQ-Linear, Methodology > Algorithmic
 * Approach: the per-bin products run backward with the transposed spectrum).
 *
 * eqlin_cyclic_weight_spectrum_adjoint writes V's spectrum.  W: device
 * [Cout][Cin][N] of `dtype` (the forward's weight).  Wspec: device buffer of at
 * least eqlin_cyclic_spectrum_bytes(N, Cout, Cin, dtype) bytes (note the
 * swapped channel counts), opaque.  Run once per weight.
 * eqlin_cyclic_backward_data computes dx: dy device [T][Cout][N], dx device
 * [T][Cin][N], both `dtype`; it is eqlin_cyclic_forward(dy, Wspec, dx, T, N,
 * Cout, Cin, ...) and takes the tensor-core path under that call's conditions
 * (with Cin and Cout swapped).  T = 0 is a no-op. */
EQLIN_API int eqlin_cyclic_weight_spectrum_adjoint(const void *W, int N, int Cin, int Cout, int dtype,
                                         void *Wspec, size_t Wspec_bytes, eqlin_stream_t stream);
EQLIN_API int eqlin_cyclic_backward_data(const void *dy, const void *Wspec, void *dx, int64_t T, int N,
                               int Cin, int Cout, int dtype, eqlin_stream_t stream);
EQLIN_API int eqlin_cyclic_backward_data_ex(const void *dy, const void *Wspec, void *dx, int64_t T,
                                  int N, int Cin, int Cout, int dtype, int path,
                                  eqlin_stream_t stream);

/* Weight gradient: the gradient of sum(dy * y) with respect to the shared
 * weight,
 *     dW[o, i, m] = sum_t sum_g dy[t, o, g] x[t, i, (g - m) mod N],
 * computed per frequency bin, C_k = sum_t DY_k[t, o] conj(X_k[t, i]), and
 * transformed back (the cross-correlation theorem; the backward counterpart
 * of the per-bin products of Flash EQ-Linear, Methodology > Algorithmic
 * Approach).  x: device [T][Cin][N], dy: device [T][Cout][N], dW: device
 * [Cout][Cin][N] (overwritten), all `dtype`; fp32 accumulation.
 * The tokens are split into ranges whose fp32 partial sums go to `workspace`,
 * caller-owned device memory of at least
 * eqlin_cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, dtype) bytes
 * (16-byte aligned; its contents on entry do not matter).  The partials are
 * summed in a fixed order, so the result does not depend on scheduling.
 * T = 0 writes dW = 0.  Supported: 1 <= N <= 16, any Cin, Cout >= 1.
 * Paths: for N = 8, bf16 and Cin, Cout >= 8 the per-bin products run on tensor cores (the
 * half spectra of x and dy rounded to bf16 as MMA operands, fp32
 * accumulation); everything else, and EQLIN_PATH_SIMT, on CUDA cores in fp32.
 * The workspace size covers either path.  eqlin_cyclic_weight_grad takes
 * EQLIN_PATH_AUTO; eqlin_cyclic_weight_grad_ex takes a path (EQLIN_PATH_TC for
 * a shape without a tensor-core path returns EQLIN_ERR_UNSUPPORTED). */
EQLIN_API size_t eqlin_cyclic_weight_grad_workspace_bytes(int64_t T, int N, int Cin, int Cout, int dtype);
EQLIN_API int eqlin_cyclic_weight_grad(const void *x, const void *dy, void *dW, int64_t T, int N, int Cin,
                             int Cout, int dtype, void *workspace, size_t workspace_bytes,
                             eqlin_stream_t stream);
EQLIN_API int eqlin_cyclic_weight_grad_ex(const void *x, const void *dy, void *dW, int64_t T, int N,
                                int Cin, int Cout, int dtype, void *workspace, size_t workspace_bytes,
                                int path, eqlin_stream_t stream);

/* Weight gradient without a caller workspace, for callers that cannot
 * allocate device memory (code running where cudaMalloc is not allowed or not
 * safe: inside an allocator or memory-pool callback, under a framework that
 * reserves all device memory up front, or in a plugin that must not touch the
 * device heap).  The source pages have no counterpart: this is a calling
 * convenience of this library, not part of the method.
 *
 * Same arguments, result and supported shapes as eqlin_cyclic_weight_grad
 * minus the workspace.  The per-split partial sums live in a fixed array of
 * EQLIN_NOALLOC_SCRATCH_BYTES inside the library's device image, which every
 * GPU that loads the library holds until the process exits; the call itself
 * allocates and frees nothing.  It uses as many token splits as fit there (at
 * most as many as eqlin_cyclic_weight_grad), so its summation order, and thus
 * its last bits, can differ from that function's.
 * Limits and caveats:
 *  - Cin * Cout * N * 4 must not exceed EQLIN_NOALLOC_SCRATCH_BYTES (one split
 *    must fit); larger layers return EQLIN_ERR_SIZE before any launch.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it; make that first call before any
 *    stream capture on that device.  The cached address does not survive
 *    cudaDeviceReset: after resetting a device, do not call this entry point
 *    on it again in the same process.
 *  - All calls share the one array: calls whose kernels may overlap on the GPU
 *    (different streams with no ordering between them) race and give wrong
 *    results.  Calls ordered on one stream are fine; each call writes every
 *    scratch element it reads before reading it, so the previous call's
 *    leftover contents never matter. */
#define EQLIN_NOALLOC_SCRATCH_BYTES (8u << 20)
EQLIN_API int eqlin_cyclic_weight_grad_noalloc(const void *x, const void *dy, void *dW, int64_t T, int N,
                                     int Cin, int Cout, int dtype, eqlin_stream_t stream);

/* ---------------------------------------------------------------- D8 */

/* Bytes of the packed D8 weight buffer for C channels (C % 8 == 0, C >= 8). */
EQLIN_API size_t eqlin_d8_weight_bytes(int C, int dtype);

/* Pack the Fourier-domain blocks (Quick ViTs review, Key design 2):
 * wA1, wA2, wB1, wB2: device [C/8][C/8]; wE: device [C/4][C/4], all `dtype`,
 * [out][in].  wE acts on the vector v_a[e], e = 2*i + b, where for field i the
 * E coordinates form the 2x2 matrix Z_i[a][b]; the same wE is applied for
 * a = 0 and a = 1.  Wpack: >= eqlin_d8_weight_bytes(C, dtype) bytes, opaque. */
EQLIN_API int eqlin_d8_pack_weights(const void *wA1, const void *wA2, const void *wB1, const void *wB2,
                          const void *wE, int C, int dtype, void *Wpack, size_t Wpack_bytes,
                          eqlin_stream_t stream);

/* D8 forward: per field z = Q x (8x8 orthogonal change of basis to the
 * coordinates [A1, A2, B1, B2, E00, E01, E10, E11]; Q[chi][g] = chi(g)/sqrt 8
 * for the 1-D irreps A1: r,s -> 1;  A2: r -> 1, s -> -1;  B1: r -> -1, s -> 1;
 * B2: r, s -> -1;  Q[E_ab][g] = rho_E(g)[a][b] / 2 with rho_E(r) = [[0,-1],[1,0]],
 * rho_E(s) = diag(1,-1)), the block products, y = Q^T z', then
 * y = 0.5 y (1 + erf(y / sqrt 2)) if fuse_gelu != 0.
 * x, y: device [T][C/8][8].  T = 0 is a no-op.  The tensor-core path needs
 * EQLIN_BF16 and C % 256 == 0, 256 <= C <= 1280, and y 32-byte aligned (AUTO
 * falls back to SIMT otherwise; TC returns EQLIN_ERR_ALIGN then). */
EQLIN_API int eqlin_d8_forward(const void *x, const void *Wpack, void *y, int64_t T, int C, int fuse_gelu,
                     int dtype, eqlin_stream_t stream);
EQLIN_API int eqlin_d8_forward_ex(const void *x, const void *Wpack, void *y, int64_t T, int C,
                        int fuse_gelu, int dtype, int path, eqlin_stream_t stream);
EQLIN_API int eqlin_d8_auto_path(int C, int dtype);

/* D8 layers that keep features in the Fourier domain (Quick ViTs review, Key
 * design 1: features stay in the Fourier domain between layers; Key design 2:
 * Schur blocks, E shared over its two row coordinates).  A feature z is
 * device [T][F][8] with each field's coordinates in the order
 * [A1, A2, B1, B2, E00, E01, E10, E11] (the basis of eqlin_d8_forward).
 *
 * eqlin_d8_fourier_pack_weights: wA1, wA2, wB1, wB2 device [F_out][F_in],
 * wE device [2 F_out][2 F_in] acting on v_a[e = 2i + b] = z[i][E_ab] for
 * a = 0 and a = 1 alike, all `dtype`; Wpack: caller-owned device memory of
 * eqlin_d8_fourier_weight_bytes(F_in, F_out, dtype) bytes (fp32, opaque).
 *
 * eqlin_d8_fourier_linear: y [T][F_out][8] = the block product of z
 * [T][F_in][8]; with roundtrip_gelu = 1 each output field then goes to the
 * regular domain, through GELU (exact erf form) and back:
 * y = Q GELU(Q^T blocks(z)), the MLP's pointwise nonlinearity (it must act
 * where the group permutes slots).  y must not overlap z.
 *
 * eqlin_d8_fourier_mlp: the transformer MLP in the Fourier domain,
 * y = contract(Q GELU(Q^T expand(z))), expand F -> F_hidden (W1pack, packed
 * with F_in = F, F_out = F_hidden), contract F_hidden -> F (W2pack).
 * hidden: caller-owned device [T][F_hidden][8] `dtype` buffer (overwritten;
 * intermediate values are rounded to `dtype` there).  No buffers may overlap.
 *
 * fp32, bf16 or fp16 I/O, fp32 accumulation; F_in, F_out >= 1; pointers
 * 16-byte aligned.  T = 0 does nothing.  Paths: bf16 layers with
 * F_in % 16 == 0 (16..160) and F_out % 32 == 0 run on the fused tensor-core
 * kernel (EQLIN_PATH_AUTO when y is 32-byte aligned; the pack then carries its
 * weight stages too), everything else on CUDA cores.  In the MLP block each
 * layer takes its own path: at C = 1280 (F = 160, F_hidden = 640) the
 * expansion runs on tensor cores, and the contraction too when
 * eqlin_d8_fourier_mlp_ws is given its workspace (else on CUDA cores).
 * eqlin_d8_fourier_linear takes EQLIN_PATH_AUTO; _ex takes a path. */
EQLIN_API size_t eqlin_d8_fourier_weight_bytes(int F_in, int F_out, int dtype);
EQLIN_API int eqlin_d8_fourier_pack_weights(const void *wA1, const void *wA2, const void *wB1,
                                  const void *wB2, const void *wE, int F_in, int F_out, int dtype,
                                  void *Wpack, size_t Wpack_bytes, eqlin_stream_t stream);
EQLIN_API int eqlin_d8_fourier_linear(const void *z, const void *Wpack, void *y, int64_t T, int F_in,
                            int F_out, int roundtrip_gelu, int dtype, eqlin_stream_t stream);
EQLIN_API int eqlin_d8_fourier_linear_ex(const void *z, const void *Wpack, void *y, int64_t T, int F_in,
                               int F_out, int roundtrip_gelu, int dtype, int path, eqlin_stream_t stream);
/* Layers with F_in > 160 (bf16, F_in % 16 == 0, F_out % 32 == 0) reach the
 * tensor cores as column slices of at most 160 input fields, each run as its
 * own layer into a bf16 partial output, then summed in slice order (the GELU
 * round trip, if asked, after the sum).  The partials need a caller-owned
 * workspace of eqlin_d8_fourier_workspace_bytes(T, F_in, F_out, dtype) bytes
 * (0 when the layer needs none), 32-byte aligned, passed to the _ws forms;
 * without it such layers run on CUDA cores. */
EQLIN_API size_t eqlin_d8_fourier_workspace_bytes(int64_t T, int F_in, int F_out, int dtype);
EQLIN_API int eqlin_d8_fourier_linear_ws(const void *z, const void *Wpack, void *y, int64_t T, int F_in,
                               int F_out, int roundtrip_gelu, int dtype, int path, void *workspace,
                               size_t workspace_bytes, eqlin_stream_t stream);
EQLIN_API size_t eqlin_d8_fourier_mlp_workspace_bytes(int64_t T, int F, int F_hidden, int dtype);
EQLIN_API int eqlin_d8_fourier_mlp_ws(const void *z, const void *W1pack, const void *W2pack, void *hidden,
                            void *y, int64_t T, int F, int F_hidden, int dtype, void *workspace,
                            size_t workspace_bytes, eqlin_stream_t stream);
EQLIN_API int eqlin_d8_fourier_mlp(const void *z, const void *W1pack, const void *W2pack, void *hidden,
                         void *y, int64_t T, int F, int F_hidden, int dtype, eqlin_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EQLIN_H_ */
