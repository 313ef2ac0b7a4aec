// CUDA-core (SIMT) kernels: weight-spectrum precompute, D8 weight packing and
// the general forward path for every supported shape and dtype.
//
// The SIMT forward is the bandwidth-oriented path for small channel counts,
// small or odd group sizes and fp32 I/O (a TF32 tensor core cannot hold the
// 1e-5 fp32 tolerance).  Each CTA stages a tile of tokens, transforms each
// field to its half spectrum in shared memory (fp32), then every thread
// accumulates the per-bin complex products for one output field and four
// tokens and applies the inverse transform on the way out.
#include <math.h>

#include "eqlin_internal.cuh"

namespace eqlin {

// ============================================================ spectrum

struct Twiddles {
  double c[kMaxN];  // cos(2 pi j / N)
  double s[kMaxN];  // sin(2 pi j / N)
};

// What[k, o, i] = (1/N) sum_m V[o,i,m] exp(-2 pi i m k / N), in fp64, stored
// as fp32 Ws[i][c][o] in the real-coordinate order of DftTables, for the layer
// Cin -> Cout whose weight V is
//   adjoint = 0: V = W, W stored [Cout][Cin][N];
//   adjoint = 1: V[o,i,m] = W[i,o,(-m) mod N], W stored [Cin][Cout][N] (the
//                weight of the backward data pass of the layer W: Cout -> Cin;
//                its spectrum is the conjugate transpose of W's).
template <typename T>
__global__ void cyclic_spectrum_simt_kernel(const T *__restrict__ W, int N, int Cin, int Cout,
                                            int adjoint, Twiddles tw, float *__restrict__ Ws) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= Cin * Cout) return;
  const int o = idx % Cout;
  const int i = idx / Cout;
  double w[kMaxN];
  for (int m = 0; m < N; ++m)
    w[m] = (double)to_f32(adjoint ? W[((size_t)i * Cout + o) * N + (N - m) % N]
                                  : W[((size_t)o * Cin + i) * N + m]);
  const double invN = 1.0 / (double)N;
  const int half = N / 2;
  for (int k = 0; k <= half; ++k) {
    double re = 0.0, im = 0.0;
    for (int m = 0; m < N; ++m) {
      const int j = (m * k) % N;
      re += w[m] * tw.c[j];
      im -= w[m] * tw.s[j];
    }
    re *= invN;
    im *= invN;
    if (k == 0) {
      Ws[((size_t)i * N + 0) * Cout + o] = (float)re;
    } else if (2 * k == N) {
      Ws[((size_t)i * N + (N - 1)) * Cout + o] = (float)re;
    } else {
      Ws[((size_t)i * N + (2 * k - 1)) * Cout + o] = (float)re;
      Ws[((size_t)i * N + (2 * k)) * Cout + o] = (float)im;
    }
  }
}

int launch_cyclic_spectrum(const void *W, int N, int Cin, int Cout, int dtype, int adjoint,
                           void *Wspec, const CyclicSpecLayout &L, cudaStream_t s) {
  Twiddles tw;
  for (int j = 0; j < kMaxN; ++j) {
    tw.c[j] = tw.s[j] = 0.0;
    if (j < N) unit_root(j, N, &tw.c[j], &tw.s[j]);
  }
  float *Ws = reinterpret_cast<float *>(static_cast<char *>(Wspec) + L.simt_offset);
  const int n = Cin * Cout;
  const int threads = 256;
  const int blocks = (n + threads - 1) / threads;
  if (dtype == EQLIN_F32)
    cyclic_spectrum_simt_kernel<float><<<blocks, threads, 0, s>>>(
        static_cast<const float *>(W), N, Cin, Cout, adjoint, tw, Ws);
  else if (dtype == EQLIN_F16)
    cyclic_spectrum_simt_kernel<__half><<<blocks, threads, 0, s>>>(
        static_cast<const __half *>(W), N, Cin, Cout, adjoint, tw, Ws);
  else
    cyclic_spectrum_simt_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(W), N, Cin, Cout, adjoint, tw, Ws);
  int rc = check_launch("cyclic spectrum (simt section)");
  if (rc != EQLIN_OK) return rc;
  if (L.tc_bytes) {
    char *tc = static_cast<char *>(Wspec) + L.tc_offset;
    rc = N == 16 ? launch_cyclic16_tc_pack(W, Cin, Cout, adjoint, tc, s)
         : N == 4 ? launch_cyclic4_tc_pack(W, Cin, Cout, adjoint, tc, s)
         : dtype == EQLIN_F32 ? launch_cyclic_tc_f32_pack(W, Cin, Cout, adjoint, tc, s)
                  : launch_cyclic_tc_pack(W, N, Cin, Cout, adjoint, dtype, tc, s);
    if (rc != EQLIN_OK) return rc;
  }
  return EQLIN_OK;
}

// ============================================================ cyclic forward

constexpr int kSimtThreads = 256;  // 8 warps
constexpr int kSimtTT = 32;        // tokens per CTA (4 per thread)
constexpr int kSimtTPT = 4;        // tokens per thread
constexpr int kSimtIC = 16;        // input fields per shared-memory chunk
constexpr int kSimtOT = 32;        // output fields per CTA (one per lane)

template <int N, typename T>
__global__ void __launch_bounds__(kSimtThreads)
cyclic_forward_simt_kernel(const T *__restrict__ x, const float *__restrict__ Ws,
                           T *__restrict__ y, int64_t Tn, int Cin, int Cout, DftTables tab) {
  __shared__ float Xs[kSimtTT][kSimtIC][N + 1];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kSimtTT;
  const int o = blockIdx.y * kSimtOT + lane;

  float acc[kSimtTPT][N];
#pragma unroll
  for (int a = 0; a < kSimtTPT; ++a)
#pragma unroll
    for (int c = 0; c < N; ++c) acc[a][c] = 0.f;

  for (int i0 = 0; i0 < Cin; i0 += kSimtIC) {
    __syncthreads();
    // forward real DFT of each (token, field) of the chunk into shared memory
    for (int p = threadIdx.x; p < kSimtTT * kSimtIC; p += kSimtThreads) {
      const int tl = p / kSimtIC;
      const int il = p % kSimtIC;
      const int64_t t = t0 + tl;
      const int i = i0 + il;
      float v[N];
      if (t < Tn && i < Cin) {
        load_field<N, T>(x + ((size_t)t * Cin + i) * N, v);
      } else {
#pragma unroll
        for (int h = 0; h < N; ++h) v[h] = 0.f;
      }
      if constexpr (N == 4) {
        p4_forward(v, Xs[tl][il]);
      } else {
#pragma unroll
        for (int c = 0; c < N; ++c) {
          float sacc = 0.f;
#pragma unroll
          for (int h = 0; h < N; ++h) sacc = fmaf(tab.fwd[c][h], v[h], sacc);
          Xs[tl][il][c] = sacc;
        }
      }
    }
    __syncthreads();
    if (o < Cout) {
      const int iend = min(kSimtIC, Cin - i0);
      for (int il = 0; il < iend; ++il) {
        float w[N];
        const float *wp = Ws + ((size_t)(i0 + il) * N) * Cout + o;
#pragma unroll
        for (int c = 0; c < N; ++c) w[c] = __ldg(wp + (size_t)c * Cout);
#pragma unroll
        for (int a = 0; a < kSimtTPT; ++a) {
          const float *X = Xs[warp * kSimtTPT + a][il];
          acc[a][0] = fmaf(w[0], X[0], acc[a][0]);
#pragma unroll
          for (int k = 1; 2 * k < N; ++k) {
            const int cr = 2 * k - 1, ci = 2 * k;
            acc[a][cr] = fmaf(w[cr], X[cr], fmaf(-w[ci], X[ci], acc[a][cr]));
            acc[a][ci] = fmaf(w[cr], X[ci], fmaf(w[ci], X[cr], acc[a][ci]));
          }
          if (N % 2 == 0 && N > 1) acc[a][N - 1] = fmaf(w[N - 1], X[N - 1], acc[a][N - 1]);
        }
      }
    }
  }
  if (o >= Cout) return;
  // inverse real DFT and store
#pragma unroll
  for (int a = 0; a < kSimtTPT; ++a) {
    const int64_t t = t0 + warp * kSimtTPT + a;
    if (t >= Tn) continue;
    T *dst = y + ((size_t)t * Cout + o) * N;
    float yv[N];
    if constexpr (N == 4) {
      p4_inverse(acc[a], yv);
    } else {
#pragma unroll
      for (int g = 0; g < N; ++g) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < N; ++c) s = fmaf(tab.inv[g][c], acc[a][c], s);
        yv[g] = s;
      }
    }
    store_field<N, T>(dst, yv);   // lanes hold consecutive output fields: one contiguous span
  }
}

template <typename T>
static int dispatch_cyclic_simt(const T *x, const float *Ws, T *y, int64_t Tn, int N, int Cin,
                                int Cout, const DftTables &tab, cudaStream_t s) {
  const int64_t gx = (Tn + kSimtTT - 1) / kSimtTT;
  if (gx > 0x7fffffffLL) return set_error(EQLIN_ERR_UNSUPPORTED, "T too large for the SIMT grid");
  dim3 grid((unsigned)gx, (unsigned)((Cout + kSimtOT - 1) / kSimtOT));
  if (grid.y > 65535) return set_error(EQLIN_ERR_UNSUPPORTED, "Cout too large for the SIMT grid");
  switch (N) {
#define EQLIN_CASE(NN)                                                                  \
  case NN:                                                                              \
    cyclic_forward_simt_kernel<NN, T><<<grid, kSimtThreads, 0, s>>>(x, Ws, y, Tn, Cin,   \
                                                                    Cout, tab);         \
    break;
    EQLIN_CASE(1) EQLIN_CASE(2) EQLIN_CASE(3) EQLIN_CASE(4) EQLIN_CASE(5) EQLIN_CASE(6)
    EQLIN_CASE(7) EQLIN_CASE(8) EQLIN_CASE(9) EQLIN_CASE(10) EQLIN_CASE(11) EQLIN_CASE(12)
    EQLIN_CASE(13) EQLIN_CASE(14) EQLIN_CASE(15) EQLIN_CASE(16)
#undef EQLIN_CASE
    default:
      return set_error(EQLIN_ERR_UNSUPPORTED, "N=%d not in 1..16", N);
  }
  return check_launch("cyclic forward (simt)");
}

int launch_cyclic_simt(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                       int Cout, int dtype, const CyclicSpecLayout &L, cudaStream_t s) {
  DftTables tab;
  make_dft_tables(N, &tab);
  const float *Ws =
      reinterpret_cast<const float *>(static_cast<const char *>(Wspec) + L.simt_offset);
  if (dtype == EQLIN_F32)
    return dispatch_cyclic_simt(static_cast<const float *>(x), Ws, static_cast<float *>(y), T, N,
                                Cin, Cout, tab, s);
  if (dtype == EQLIN_F16)
    return dispatch_cyclic_simt(static_cast<const __half *>(x), Ws, static_cast<__half *>(y), T, N,
                                Cin, Cout, tab, s);
  return dispatch_cyclic_simt(static_cast<const __nv_bfloat16 *>(x), Ws,
                              static_cast<__nv_bfloat16 *>(y), T, N, Cin, Cout, tab, s);
}

// ============================================================ D8

// SIMT section of the D8 pack: W1[c][i][o] = w_c[o][i] (c < 4, F x F each),
// then WEt[e][e2] = wE[e2][e] (2F x 2F), all fp32.
template <typename T>
__global__ void d8_pack_simt_kernel(const T *__restrict__ a1, const T *__restrict__ a2,
                                    const T *__restrict__ b1, const T *__restrict__ b2,
                                    const T *__restrict__ wE, int F, float *__restrict__ dst) {
  const int64_t n1 = (int64_t)F * F;
  const int64_t nE = 4 * n1;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < 4 * n1) {
    const int c = (int)(idx / n1);
    const int64_t r = idx % n1;
    const int i = (int)(r / F), o = (int)(r % F);
    const T *src = c == 0 ? a1 : c == 1 ? a2 : c == 2 ? b1 : b2;
    dst[idx] = to_f32(src[(size_t)o * F + i]);
  } else if (idx < 4 * n1 + nE) {
    const int64_t r = idx - 4 * n1;
    const int e = (int)(r / (2 * F)), e2 = (int)(r % (2 * F));
    dst[idx] = to_f32(wE[(size_t)e2 * (2 * F) + e]);
  }
}

int launch_d8_pack(const void *const w[5], int C, int dtype, void *Wpack, const D8PackLayout &L,
                   cudaStream_t s) {
  const int F = C / 8;
  float *dst = reinterpret_cast<float *>(static_cast<char *>(Wpack) + L.simt_offset);
  const int64_t n = 8LL * F * F;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (dtype == EQLIN_F32)
    d8_pack_simt_kernel<float><<<blocks, threads, 0, s>>>(
        (const float *)w[0], (const float *)w[1], (const float *)w[2], (const float *)w[3],
        (const float *)w[4], F, dst);
  else if (dtype == EQLIN_F16)
    d8_pack_simt_kernel<__half><<<blocks, threads, 0, s>>>(
        (const __half *)w[0], (const __half *)w[1], (const __half *)w[2], (const __half *)w[3],
        (const __half *)w[4], F, dst);
  else
    d8_pack_simt_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        (const __nv_bfloat16 *)w[0], (const __nv_bfloat16 *)w[1], (const __nv_bfloat16 *)w[2],
        (const __nv_bfloat16 *)w[3], (const __nv_bfloat16 *)w[4], F, dst);
  int rc = check_launch("d8 pack (simt section)");
  if (rc != EQLIN_OK) return rc;
  if (L.tc_bytes) {
    rc = launch_d8_tc_pack(w, C, static_cast<char *>(Wpack) + L.tc_offset, s);
    if (rc != EQLIN_OK) return rc;
  }
  return EQLIN_OK;
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752440f));
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
d8_forward_simt_kernel(const T *__restrict__ x, const float *__restrict__ W1,
                       const float *__restrict__ WEt, T *__restrict__ y, int64_t Tn, int F,
                       int gelu, D8Tables tab) {
  __shared__ float Zs[kSimtTT][kSimtIC][9];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kSimtTT;
  const int o = blockIdx.y * kSimtOT + lane;
  const size_t n1 = (size_t)F * F;

  float acc[kSimtTPT][8];
#pragma unroll
  for (int a = 0; a < kSimtTPT; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;

  for (int i0 = 0; i0 < F; i0 += kSimtIC) {
    __syncthreads();
    for (int p = threadIdx.x; p < kSimtTT * kSimtIC; p += kSimtThreads) {
      const int tl = p / kSimtIC, il = p % kSimtIC;
      const int64_t t = t0 + tl;
      const int i = i0 + il;
      float v[8];
      if (t < Tn && i < F) {
        load_field<8, T>(x + ((size_t)t * F + i) * 8, v);
      } else {
#pragma unroll
        for (int h = 0; h < 8; ++h) v[h] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float sacc = 0.f;
#pragma unroll
        for (int h = 0; h < 8; ++h) sacc = fmaf(tab.q[c][h], v[h], sacc);
        Zs[tl][il][c] = sacc;
      }
    }
    __syncthreads();
    if (o < F) {
      const int iend = min(kSimtIC, F - i0);
      for (int il = 0; il < iend; ++il) {
        const int i = i0 + il;
        float w[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = __ldg(W1 + c * n1 + (size_t)i * F + o);
        // wE^T rows e = 2i+b, columns e2 = 2o+b2
        const float2 e0 = __ldg(reinterpret_cast<const float2 *>(WEt + (size_t)(2 * i) * (2 * F) + 2 * o));
        const float2 e1 = __ldg(reinterpret_cast<const float2 *>(WEt + (size_t)(2 * i + 1) * (2 * F) + 2 * o));
#pragma unroll
        for (int a = 0; a < kSimtTPT; ++a) {
          const float *z = Zs[warp * kSimtTPT + a][il];
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(w[c], z[c], acc[a][c]);
#pragma unroll
          for (int ra = 0; ra < 2; ++ra) {
            const float zb0 = z[4 + 2 * ra + 0], zb1 = z[4 + 2 * ra + 1];
            acc[a][4 + 2 * ra + 0] = fmaf(e0.x, zb0, fmaf(e1.x, zb1, acc[a][4 + 2 * ra + 0]));
            acc[a][4 + 2 * ra + 1] = fmaf(e0.y, zb0, fmaf(e1.y, zb1, acc[a][4 + 2 * ra + 1]));
          }
        }
      }
    }
  }
  if (o >= F) return;
#pragma unroll
  for (int a = 0; a < kSimtTPT; ++a) {
    const int64_t t = t0 + warp * kSimtTPT + a;
    if (t >= Tn) continue;
    float yv[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) s = fmaf(tab.q[c][g], acc[a][c], s);
      yv[g] = gelu ? gelu_erf(s) : s;
    }
    store_field<8, T>(y + ((size_t)t * F + o) * 8, yv);
  }
}

int launch_d8_simt(const void *x, const void *Wpack, void *y, int64_t T, int C, int gelu,
                   int dtype, const D8PackLayout &L, cudaStream_t s) {
  const int F = C / 8;
  D8Tables tab;
  make_d8_tables(&tab);
  const float *W1 =
      reinterpret_cast<const float *>(static_cast<const char *>(Wpack) + L.simt_offset);
  const float *WEt = W1 + 4 * (size_t)F * F;
  const int64_t gx = (T + kSimtTT - 1) / kSimtTT;
  if (gx > 0x7fffffffLL) return set_error(EQLIN_ERR_UNSUPPORTED, "T too large for the SIMT grid");
  dim3 grid((unsigned)gx, (unsigned)((F + kSimtOT - 1) / kSimtOT));
  if (dtype == EQLIN_F32)
    d8_forward_simt_kernel<float><<<grid, kSimtThreads, 0, s>>>(
        (const float *)x, W1, WEt, (float *)y, T, F, gelu, tab);
  else if (dtype == EQLIN_F16)
    d8_forward_simt_kernel<__half><<<grid, kSimtThreads, 0, s>>>(
        (const __half *)x, W1, WEt, (__half *)y, T, F, gelu, tab);
  else
    d8_forward_simt_kernel<__nv_bfloat16><<<grid, kSimtThreads, 0, s>>>(
        (const __nv_bfloat16 *)x, W1, WEt, (__nv_bfloat16 *)y, T, F, gelu, tab);
  return check_launch("d8 forward (simt)");
}

}  // namespace eqlin
