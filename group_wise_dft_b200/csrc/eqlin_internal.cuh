// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include <type_traits>

#include "eqlin.h"

namespace eqlin {

// ----------------------------------------------------------------- errors
int set_error(int code, const char *fmt, ...);
void clear_error();   // empties this thread's eqlin_last_error() message
int check_launch(const char *what);
// dtype, N in 1..16, Cin, Cout >= 1 and Cin*N, Cout*N <= 2^24 (EQLIN_ERR_* otherwise)
int check_cyclic_shape(int N, int Cin, int Cout, int dtype);

// Device fault state: kernels whose bounded waits ran out write a nonzero code
// into a __device__ word that lives in the tensor-core translation unit (the
// first code is kept); read_device_fault() synchronises and reads (optionally
// clears) it.  Every launch of a kernel with bounded waits takes a fresh
// nonzero epoch from next_launch_epoch(), so a fault stops only the launch
// that raised it, never a later one.
int read_device_fault(int reset);
unsigned int next_launch_epoch();

enum FaultCode : unsigned int {
  FAULT_NONE = 0,
  FAULT_WAIT_X_FULL = 0x101,
  FAULT_WAIT_A_EMPTY = 0x102,
  FAULT_WAIT_A_FULL = 0x103,
  FAULT_WAIT_B_FULL = 0x104,
  FAULT_WAIT_B_EMPTY = 0x105,
  FAULT_WAIT_ACC_FULL = 0x106,
  FAULT_WAIT_ACC_EMPTY = 0x107,
  FAULT_WAIT_X_EMPTY = 0x108,
  FAULT_WAIT_PEER = 0x109,
  FAULT_WAIT_STAGE = 0x10a,
  FAULT_SELFTEST = EQLIN_FAULT_SELFTEST,
};

// ----------------------------------------------------------------- tables
// Real-coordinate order of one field's half spectrum, N real numbers:
//   c = 0            : Re X_0
//   c = 2k-1, 2k     : Re X_k, Im X_k     (1 <= k < N/2, or k <= (N-1)/2 for odd N)
//   c = N-1 (N even) : Re X_{N/2}
// Forward:  X_c = sum_h Fwd[c][h] x_h.   Inverse: y_g = sum_c Inv[g][c] Y_c
// (the 1/N of the inverse DFT lives in the weight spectrum).
constexpr int kMaxN = 16;
struct DftTables {
  float fwd[kMaxN][kMaxN];
  float inv[kMaxN][kMaxN];
};
void make_dft_tables(int N, DftTables *t);

// cos and sin of 2 pi j / N in double, exactly 0 and +-1 at whole quarter turns.
void unit_root(int j, int N, double *c, double *s);

// p4 (N = 4): the 4-point DFT's entries are 0, +-1 and +-i, so the forward
// transform and its one-sided inverse are additions (and one doubling), exact
// in floating point (Flash EQ-Linear, Specialization for p4).  Coordinates as
// above: [Re X0, Re X1, Im X1, Re X2]; X_1 = x0 - x2 + i (x3 - x1).
__host__ __device__ __forceinline__ void p4_forward(const float *v, float *X) {
  const float e = v[0] + v[2], f = v[1] + v[3];
  X[0] = e + f;
  X[1] = v[0] - v[2];
  X[2] = v[3] - v[1];
  X[3] = e - f;
}
// y_g = Y0 + (-1)^g Y2 + 2 Re(Y1 i^g) (the 1/N lives in the weight spectrum).
__host__ __device__ __forceinline__ void p4_inverse(const float *Y, float *y) {
  const float p = Y[0] + Y[3], m = Y[0] - Y[3], r = 2.0f * Y[1], i = 2.0f * Y[2];
  y[0] = p + r;
  y[1] = m - i;
  y[2] = p - r;
  y[3] = m + i;
}

// D8 change of basis, Q[c][g], coordinates [A1, A2, B1, B2, E00, E01, E10, E11].
struct D8Tables {
  float q[8][8];
};
void make_d8_tables(D8Tables *t);

// ------------------------------------------------------- spectrum layouts
// Weight-spectrum buffer = [header-free] SIMT section, then (optionally) the
// tensor-core section, each starting on a 256-byte boundary.
struct CyclicSpecLayout {
  size_t simt_offset, simt_bytes;   // fp32 Ws[i][c][o]
  size_t tc_offset, tc_bytes;       // bf16 packed B panels (0 if no TC path)
  size_t total;
};
CyclicSpecLayout cyclic_spec_layout(int N, int Cin, int Cout, int dtype);

struct D8PackLayout {
  size_t simt_offset, simt_bytes;   // fp32 W1[c][i][o] (c<4), then WEt[e][e'] = wE[e'][e]
  size_t tc_offset, tc_bytes;
  size_t total;
};
D8PackLayout d8_pack_layout(int C, int dtype);

// ------------------------------------------------------------- launchers
int launch_cyclic_spectrum(const void *W, int N, int Cin, int Cout, int dtype, int adjoint, void *Wspec,
                           const CyclicSpecLayout &L, cudaStream_t s);
int launch_cyclic_simt(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                       int Cout, int dtype, const CyclicSpecLayout &L, cudaStream_t s);
int launch_d8_pack(const void *const w[5], int C, int dtype, void *Wpack, const D8PackLayout &L,
                   cudaStream_t s);
int launch_d8_simt(const void *x, const void *Wpack, void *y, int64_t T, int C, int gelu,
                   int dtype, const D8PackLayout &L, cudaStream_t s);

// Weight gradient (simt_wgrad.cu): S token splits, fp32 partials [S][Cout][Cin][N].
int cyclic_wgrad_splits(int64_t T, int Cin, int Cout);
size_t cyclic_wgrad_part_bytes(int S, int N, int Cin, int Cout);
int launch_cyclic_wgrad(const void *x, const void *dy, void *dW, int64_t T, int N, int Cin,
                        int Cout, int dtype, float *part, int S, cudaStream_t s);
// The second pass alone: dW from S partials (fixed order), any dtype.
int launch_cyclic_wgrad_finish(const float *part, int S, int N, int Cin, int Cout, int dtype, void *dW,
                               cudaStream_t s);

// Weight gradient on tensor cores (wgrad_tc.cu), C_8 and bf16: fills the same
// [S][Cout][Cin][8] partials, finished by launch_cyclic_wgrad_finish.
struct WgradTcPlan {
  int n_ot, n_it, ntile;       // 128-field tiles of the output and input fields
  int splits;                  // S, token splits
  int tokens_per_split;
};
bool cyclic_wgrad_tc_supported(int64_t T, int N, int Cin, int Cout, int dtype);
WgradTcPlan cyclic_wgrad_tc_plan(int64_t T, int Cin, int Cout);
int launch_cyclic_wgrad_tc_partials(const void *x, const void *dy, float *part, int64_t T, int Cin,
                                    int Cout, const WgradTcPlan &plan, cudaStream_t s);

// D8 layers in the Fourier domain (d8_fourier.cu): fp32 pack W1[c][i][o], WEt[e][e'].
size_t d8_fourier_pack_bytes(int F_in, int F_out);
int launch_d8_fourier_pack(const void *const w[5], int F_in, int F_out, int dtype, void *Wpack,
                           cudaStream_t s);
int launch_d8_fourier_linear(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                             int gelu, int dtype, cudaStream_t s);
// y = sum over S bf16 partials [S][T][F_out][8] (+ the GELU round trip), bf16.
int launch_d8_slice_sum(const void *parts, int S, int64_t T, int F_out, int roundtrip_gelu, void *y,
                        cudaStream_t s);

// Bounded-wait self-test (spectral_tc.cu, beside the fault word).
int launch_bounded_wait_selftest(uint64_t limit_ns, int arrive, unsigned long long *elapsed_ns,
                                 cudaStream_t s);

// Tensor-core path (spectral_tc.cu)
bool cyclic_tc_supported(int N, int Cin, int Cout, int dtype);
bool d8_tc_supported(int C, int dtype);
size_t cyclic_tc_bytes(int N, int Cin, int Cout);
size_t d8_tc_bytes(int C);
int launch_cyclic_tc_pack(const void *W, int N, int Cin, int Cout, int adjoint, int dtype, void *dst,
                          cudaStream_t s);
int launch_d8_tc_pack(const void *const w[5], int C, void *dst, cudaStream_t s);
int launch_cyclic_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout, int dtype,
                     cudaStream_t s);
// fp16 I/O on the fused kernel (fp16 spectra and weights as the MMA operands):
// taken only when asked for (EQLIN_PATH_TC), not by EQLIN_PATH_AUTO.
bool cyclic_tc_f16_supported(int N, int Cin, int Cout, int dtype);
// p4 (C_4, bf16) on the fused kernel, as pairs of C_4 fields; taken only when
// asked for (EQLIN_PATH_TC).
// fp32 C_8 at about 1e-5 on the bf16 MMAs (split spectra, a 3 Cin-wide layer;
// Cin 16, 32 or 48): a workspace for the split activations; PATH_TC only.
bool cyclic_tc_f32_supported(int N, int Cin, int Cout, int dtype);
size_t cyclic_tc_f32_bytes(int Cin, int Cout);
size_t cyclic_tc_f32_workspace_bytes(int64_t T, int Cin, int Cout);
int launch_cyclic_tc_f32_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s);
int launch_cyclic_tc_f32(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                         void *workspace, cudaStream_t s);
bool cyclic4_tc_supported(int N, int Cin, int Cout, int dtype);
size_t cyclic4_tc_bytes(int Cin, int Cout);
int launch_cyclic4_tc_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s);
int launch_cyclic4_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout, cudaStream_t s);
int launch_d8_tc(const void *x, const void *Bpack, void *y, int64_t T, int C, int gelu,
                 cudaStream_t s);
// Fourier-domain D8 layer F_in -> F_out on the fused kernel (input and output
// in coordinates; roundtrip_gelu: Q GELU(Q^T .) on the output).
bool d8_fourier_tc_supported(int F_in, int F_out, int dtype);
size_t d8_fourier_tc_bytes(int F_in, int F_out);
// A layer of F_slice input fields cut from blocks F_total wide at column k0
// (k0 = 0, F_slice = F_total: the whole layer); z rows are z_ld fields apart.
int launch_d8_fourier_tc_pack(const void *const w[5], int F_total, int k0, int F_slice, int F_out,
                              void *dst, cudaStream_t s);
int launch_d8_fourier_tc(const void *z, const void *Bpack, void *y, int64_t T, int F_in, int F_out,
                         int roundtrip_gelu, int z_ld, cudaStream_t s);
// C_16 on the tensor-core kernel in two passes (even cyclic, odd negacyclic halves)
bool cyclic16_tc_supported(int Cin, int Cout, int dtype);
size_t cyclic16_tc_bytes(int Cin, int Cout);
size_t cyclic16_tc_workspace_bytes(int64_t T, int Cin, int Cout);
int launch_cyclic16_tc_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s);
int launch_cyclic16_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                       void *workspace, cudaStream_t s);

// ---------------------------------------------------------------- device helpers
template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) {
  return __half2float(v);
}
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) {
  return __float2half_rn(v);
}

// One field's N contiguous elements of type T, moved as the widest vectors
// (16, 8 or 4 bytes) that N * sizeof(T) allows; the field's address is
// field-index * N * sizeof(T) past a 16-byte aligned base, so every vector is
// aligned.  Lanes that handle consecutive fields then touch one contiguous
// span per instruction.
template <int N, typename T>
__device__ __forceinline__ void load_field(const T *__restrict__ src, float (&v)[N]) {
  constexpr int B = N * (int)sizeof(T);
  constexpr int V = B % 16 == 0 ? 16 : (B % 8 == 0 ? 8 : (B % 4 == 0 ? 4 : 0));
  if constexpr (V == 0) {
#pragma unroll
    for (int h = 0; h < N; ++h) v[h] = to_f32(src[h]);
  } else {
    constexpr int E = V / (int)sizeof(T);   // elements per vector
    using Vec = typename std::conditional<V == 16, uint4, typename std::conditional<V == 8, uint2, uint32_t>::type>::type;
#pragma unroll
    for (int j = 0; j < B / V; ++j) {
      union { Vec q; T e[E]; } u;
      u.q = __ldg(reinterpret_cast<const Vec *>(src) + j);
#pragma unroll
      for (int k = 0; k < E; ++k) v[j * E + k] = to_f32(u.e[k]);
    }
  }
}

template <int N, typename T>
__device__ __forceinline__ void store_field(T *__restrict__ dst, const float (&v)[N]) {
  constexpr int B = N * (int)sizeof(T);
  constexpr int V = B % 16 == 0 ? 16 : (B % 8 == 0 ? 8 : (B % 4 == 0 ? 4 : 0));
  if constexpr (V == 0) {
#pragma unroll
    for (int g = 0; g < N; ++g) dst[g] = from_f32<T>(v[g]);
  } else {
    constexpr int E = V / (int)sizeof(T);
    using Vec = typename std::conditional<V == 16, uint4, typename std::conditional<V == 8, uint2, uint32_t>::type>::type;
#pragma unroll
    for (int j = 0; j < B / V; ++j) {
      union { Vec q; T e[E]; } u;
#pragma unroll
      for (int k = 0; k < E; ++k) u.e[k] = from_f32<T>(v[j * E + k]);
      reinterpret_cast<Vec *>(dst)[j] = u.q;
    }
  }
}

}  // namespace eqlin
