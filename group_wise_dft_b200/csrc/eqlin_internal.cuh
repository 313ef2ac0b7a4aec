// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "eqlin.h"

namespace eqlin {

// ----------------------------------------------------------------- errors
int set_error(int code, const char *fmt, ...);
int check_launch(const char *what);

// Device fault word: kernels whose bounded waits ran out write a nonzero code
// into a __device__ word that lives in the tensor-core translation unit;
// read_device_fault() synchronises and reads (optionally clears) it.
int read_device_fault(int reset);

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

// Bounded-wait self-test (spectral_tc.cu, beside the fault word).
int launch_bounded_wait_selftest(uint64_t limit_ns, int arrive, unsigned long long *elapsed_ns,
                                 cudaStream_t s);

// Tensor-core path (spectral_tc.cu)
bool cyclic_tc_supported(int N, int Cin, int Cout, int dtype);
bool d8_tc_supported(int C, int dtype);
size_t cyclic_tc_bytes(int N, int Cin, int Cout);
size_t d8_tc_bytes(int C);
int launch_cyclic_tc_pack(const void *W, int N, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s);
int launch_d8_tc_pack(const void *const w[5], int C, void *dst, cudaStream_t s);
int launch_cyclic_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                     cudaStream_t s);
int launch_d8_tc(const void *x, const void *Bpack, void *y, int64_t T, int C, int gelu,
                 cudaStream_t s);

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

}  // namespace eqlin
