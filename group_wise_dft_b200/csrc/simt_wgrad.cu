// Weight gradient of the cyclic layer, on CUDA cores.
//
// For y[t,o,g] = sum_i sum_h W[o,i,(g-h) mod N] x[t,i,h], the gradient of
// sum(dy * y) with respect to the shared weight is the token sum of a circular
// cross-correlation,
//     dW[o,i,m] = sum_t sum_g dy[t,o,g] x[t,i,(g-m) mod N],
// which the cross-correlation theorem turns into a per-bin product summed over
// tokens (the backward counterpart of Flash EQ-Linear, Methodology >
// Algorithmic Approach):
//     C_k[o,i] = sum_t DY_k[t,o] conj(X_k[t,i]),   k = 0 .. floor(N/2),
//     dW[o,i,m] = (1/N) (C_0 + (-1)^m C_{N/2} + 2 sum_{0<k<N/2} Re(C_k e^{2 pi i m k / N})).
//
// Pass 1 splits the tokens into S ranges; a CTA transforms a tile of tokens'
// x and dy fields to half spectra in shared memory (fp32) and accumulates C
// for a 32 x 32 tile of (output field, input field) pairs over its range,
// writing one fp32 partial per split into the caller's workspace.  Pass 2
// sums the S partials in a fixed order (the result does not depend on
// scheduling) and applies the inverse transform.
#include "eqlin_internal.cuh"

namespace eqlin {

namespace {

constexpr int kWgTile = 32;      // output fields and input fields per CTA
constexpr int kWgTT = 8;         // tokens per shared-memory step
constexpr int kWgThreads = 256;  // 8 warps: lane = output field, warp = 4 input fields
constexpr int kWgPairs = kWgTile * kWgTile / kWgThreads;
constexpr int kWgMinTokensPerSplit = 256;
constexpr int kWgTargetCtas = 2 * 148;

template <int N, typename T>
__global__ void __launch_bounds__(kWgThreads)
cyclic_wgrad_partial_kernel(const T *__restrict__ x, const T *__restrict__ dy,
                            float *__restrict__ part, int64_t Tn, int Cin, int Cout,
                            int64_t tok_per_split, DftTables tab) {
  __shared__ float Xs[kWgTT][kWgTile][N + 1];
  __shared__ float Ds[kWgTT][kWgTile][N + 1];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int o0 = blockIdx.x * kWgTile;
  const int i0 = blockIdx.y * kWgTile;
  const int64_t t_begin = (int64_t)blockIdx.z * tok_per_split;
  const int64_t t_end = t_begin + tok_per_split < Tn ? t_begin + tok_per_split : Tn;

  float acc[kWgPairs][N];
#pragma unroll
  for (int p = 0; p < kWgPairs; ++p)
#pragma unroll
    for (int c = 0; c < N; ++c) acc[p][c] = 0.f;

  for (int64_t tb = t_begin; tb < t_end; tb += kWgTT) {
    __syncthreads();
    // half spectra of the step's x fields (which = 0) and dy fields (which = 1)
    for (int p = threadIdx.x; p < 2 * kWgTT * kWgTile; p += kWgThreads) {
      const int which = p / (kWgTT * kWgTile);
      const int q = p - which * (kWgTT * kWgTile);
      const int tt = q / kWgTile, fl = q % kWgTile;
      const int64_t t = tb + tt;
      const int F = which ? Cout : Cin;
      const int f = (which ? o0 : i0) + fl;
      float v[N];
      if (t < t_end && f < F) {
        load_field<N, T>((which ? dy : x) + ((size_t)t * F + f) * N, v);
      } else {
#pragma unroll
        for (int h = 0; h < N; ++h) v[h] = 0.f;
      }
      float *dst = which ? Ds[tt][fl] : Xs[tt][fl];
      if constexpr (N == 4) {
        p4_forward(v, dst);
      } else {
#pragma unroll
        for (int c = 0; c < N; ++c) {
          float s = 0.f;
#pragma unroll
          for (int h = 0; h < N; ++h) s = fmaf(tab.fwd[c][h], v[h], s);
          dst[c] = s;
        }
      }
    }
    __syncthreads();
#pragma unroll 2
    for (int tt = 0; tt < kWgTT; ++tt) {
      float D[N];
#pragma unroll
      for (int c = 0; c < N; ++c) D[c] = Ds[tt][lane][c];
#pragma unroll
      for (int p = 0; p < kWgPairs; ++p) {
        const float *X = Xs[tt][warp * kWgPairs + p];
        // C += DY . conj(X), per bin
        acc[p][0] = fmaf(D[0], X[0], acc[p][0]);
#pragma unroll
        for (int k = 1; 2 * k < N; ++k) {
          const int cr = 2 * k - 1, ci = 2 * k;
          acc[p][cr] = fmaf(D[cr], X[cr], fmaf(D[ci], X[ci], acc[p][cr]));
          acc[p][ci] = fmaf(D[ci], X[cr], fmaf(-D[cr], X[ci], acc[p][ci]));
        }
        if (N % 2 == 0 && N > 1) acc[p][N - 1] = fmaf(D[N - 1], X[N - 1], acc[p][N - 1]);
      }
    }
  }
  const int o = o0 + lane;
  if (o >= Cout) return;
#pragma unroll
  for (int p = 0; p < kWgPairs; ++p) {
    const int i = i0 + warp * kWgPairs + p;
    if (i >= Cin) continue;
    float *dst = part + (((size_t)blockIdx.z * Cout + o) * Cin + i) * N;
#pragma unroll
    for (int c = 0; c < N; ++c) dst[c] = acc[p][c];
  }
}

// dW[o,i,m] = (1/N) sum_c Inv[m][c] C[c], C = sum over the S partials in order.
// One thread per (o, i); its N coordinates of a partial are moved as vectors
// (load_field) and four partials are in flight at a time, so the reduction
// streams the partials instead of waiting on one scalar load after another.
template <int N, typename T>
__global__ void cyclic_wgrad_finish_kernel(const float *__restrict__ part, int S, int Cin, int Cout,
                                           DftTables tab, T *__restrict__ dW) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)Cin * Cout) return;
  const size_t stride = (size_t)Cin * Cout * N;   // floats between consecutive partials
  const float *src = part + (size_t)idx * N;
  float C[N];
#pragma unroll
  for (int c = 0; c < N; ++c) C[c] = 0.f;
  int s = 0;
  for (; s + 4 <= S; s += 4) {
    float v[4][N];
#pragma unroll
    for (int u = 0; u < 4; ++u) load_field<N, float>(src + (size_t)(s + u) * stride, v[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int c = 0; c < N; ++c) C[c] += v[u][c];   // the partials in order, as before
  }
  for (; s < S; ++s) {
    float v[N];
    load_field<N, float>(src + (size_t)s * stride, v);
#pragma unroll
    for (int c = 0; c < N; ++c) C[c] += v[c];
  }
  const float invN = 1.0f / (float)N;
  float w[N];
  if constexpr (N == 4) {
    p4_inverse(C, w);
#pragma unroll
    for (int m = 0; m < 4; ++m) w[m] *= invN;
  } else {
#pragma unroll
    for (int m = 0; m < N; ++m) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < N; ++c) acc = fmaf(tab.inv[m][c], C[c], acc);
      w[m] = acc * invN;
    }
  }
  store_field<N, T>(dW + (size_t)idx * N, w);
}

template <typename T>
int launch_finish(const float *part, int S, int N, int Cin, int Cout, const DftTables &tab, T *dW,
                  cudaStream_t s) {
  const int64_t n = (int64_t)Cin * Cout;
  const unsigned grid = (unsigned)((n + 255) / 256);
  switch (N) {
#define EQLIN_CASE(NN)                                                                              \
  case NN:                                                                                          \
    cyclic_wgrad_finish_kernel<NN, T><<<grid, 256, 0, s>>>(part, S, Cin, Cout, tab, dW);            \
    break;
    EQLIN_CASE(1) EQLIN_CASE(2) EQLIN_CASE(3) EQLIN_CASE(4) EQLIN_CASE(5) EQLIN_CASE(6)
    EQLIN_CASE(7) EQLIN_CASE(8) EQLIN_CASE(9) EQLIN_CASE(10) EQLIN_CASE(11) EQLIN_CASE(12)
    EQLIN_CASE(13) EQLIN_CASE(14) EQLIN_CASE(15) EQLIN_CASE(16)
#undef EQLIN_CASE
    default:
      return set_error(EQLIN_ERR_UNSUPPORTED, "N=%d not in 1..16", N);
  }
  return check_launch("cyclic weight gradient (reduction)");
}

template <typename T>
int dispatch_wgrad(const T *x, const T *dy, T *dW, float *part, int S, int64_t Tn, int N, int Cin,
                   int Cout, cudaStream_t s) {
  DftTables tab;
  make_dft_tables(N, &tab);
  if (S > 0) {
    const int64_t per = (Tn + S - 1) / S;
    dim3 grid((unsigned)((Cout + kWgTile - 1) / kWgTile), (unsigned)((Cin + kWgTile - 1) / kWgTile),
              (unsigned)S);
    switch (N) {
#define EQLIN_CASE(NN)                                                                       \
  case NN:                                                                                   \
    cyclic_wgrad_partial_kernel<NN, T><<<grid, kWgThreads, 0, s>>>(x, dy, part, Tn, Cin, Cout, \
                                                                   per, tab);                \
    break;
      EQLIN_CASE(1) EQLIN_CASE(2) EQLIN_CASE(3) EQLIN_CASE(4) EQLIN_CASE(5) EQLIN_CASE(6)
      EQLIN_CASE(7) EQLIN_CASE(8) EQLIN_CASE(9) EQLIN_CASE(10) EQLIN_CASE(11) EQLIN_CASE(12)
      EQLIN_CASE(13) EQLIN_CASE(14) EQLIN_CASE(15) EQLIN_CASE(16)
#undef EQLIN_CASE
      default:
        return set_error(EQLIN_ERR_UNSUPPORTED, "N=%d not in 1..16", N);
    }
    const int rc = check_launch("cyclic weight gradient (partials)");
    if (rc != EQLIN_OK) return rc;
  }
  return launch_finish(part, S, N, Cin, Cout, tab, dW, s);
}

template <typename T>
int dispatch_finish(const float *part, int S, int N, int Cin, int Cout, T *dW, cudaStream_t s) {
  DftTables tab;
  make_dft_tables(N, &tab);
  return launch_finish(part, S, N, Cin, Cout, tab, dW, s);
}

}  // namespace

int launch_cyclic_wgrad_finish(const float *part, int S, int N, int Cin, int Cout, int dtype, void *dW,
                               cudaStream_t s) {
  if (dtype == EQLIN_F32) return dispatch_finish(part, S, N, Cin, Cout, static_cast<float *>(dW), s);
  if (dtype == EQLIN_F16) return dispatch_finish(part, S, N, Cin, Cout, static_cast<__half *>(dW), s);
  return dispatch_finish(part, S, N, Cin, Cout, static_cast<__nv_bfloat16 *>(dW), s);
}

int cyclic_wgrad_splits(int64_t T, int Cin, int Cout) {
  if (T <= 0) return 0;
  const int64_t tiles = (int64_t)((Cout + kWgTile - 1) / kWgTile) * ((Cin + kWgTile - 1) / kWgTile);
  int64_t S = (kWgTargetCtas + tiles - 1) / tiles;
  const int64_t by_tokens = (T + kWgMinTokensPerSplit - 1) / kWgMinTokensPerSplit;
  if (S > by_tokens) S = by_tokens;
  if (S < 1) S = 1;
  if (S > 65535) S = 65535;
  return (int)S;
}

size_t cyclic_wgrad_part_bytes(int S, int N, int Cin, int Cout) {
  return (size_t)S * (size_t)Cin * (size_t)Cout * (size_t)N * sizeof(float);
}

int launch_cyclic_wgrad(const void *x, const void *dy, void *dW, int64_t T, int N, int Cin,
                        int Cout, int dtype, float *part, int S, cudaStream_t s) {
  if ((Cin + kWgTile - 1) / kWgTile > 65535 || (Cout + kWgTile - 1) / kWgTile > 0x7fffffff)
    return set_error(EQLIN_ERR_UNSUPPORTED, "channel count too large for the weight-gradient grid");
  if (dtype == EQLIN_F32)
    return dispatch_wgrad(static_cast<const float *>(x), static_cast<const float *>(dy),
                          static_cast<float *>(dW), part, S, T, N, Cin, Cout, s);
  if (dtype == EQLIN_F16)
    return dispatch_wgrad(static_cast<const __half *>(x), static_cast<const __half *>(dy),
                          static_cast<__half *>(dW), part, S, T, N, Cin, Cout, s);
  return dispatch_wgrad(static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(dy),
                        static_cast<__nv_bfloat16 *>(dW), part, S, T, N, Cin, Cout, s);
}

}  // namespace eqlin
