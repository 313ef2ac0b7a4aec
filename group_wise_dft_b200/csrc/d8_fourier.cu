// D8 layers that keep their features in the Fourier domain, on CUDA cores.
//
// The Quick ViTs review (Key design 1) keeps features in the Fourier domain
// between layers: each field holds its 8 coordinates in the irreps
// [A1, A2, B1, B2, E00, E01, E10, E11] instead of the 8 regular slots.  A
// linear layer is then the Schur block product alone (Key design 2): four
// [F_out x F_in] matrices on the 1-D irreps and one [2 F_out x 2 F_in] matrix
// on E, shared by its two row coordinates a = 0, 1 (vector index e = 2i + b).
// The pointwise nonlinearity must act in the regular domain, where the group
// permutes slots, so the MLP's GELU is a round trip per field:
// z -> Q GELU(Q^T z).  The MLP block is expand (F -> F_hidden, with the round
// trip fused into its output) followed by contract (F_hidden -> F).
//
// One thread block covers 32 tokens x 32 output fields (one output field per
// lane, 4 tokens per thread); input fields stream through shared memory in
// chunks of 16 (all 8 coordinates each).  Accumulation in fp32.
#include "eqlin_internal.cuh"

namespace eqlin {
namespace {

constexpr int kFzThreads = 256;
constexpr int kFzTT = 32;   // tokens per block
constexpr int kFzTPT = 4;   // tokens per thread
constexpr int kFzIC = 16;   // input fields per chunk
constexpr int kFzOT = 32;   // output fields per block

// Weight pack (fp32): W1[c][i][o] = w_c[o][i] for c < 4 (F_in x F_out each),
// then WEt[e][e'] = wE[e'][e] (2 F_in x 2 F_out).
template <typename T>
__global__ void d8_fourier_pack_kernel(const T *__restrict__ a1, const T *__restrict__ a2,
                                       const T *__restrict__ b1, const T *__restrict__ b2,
                                       const T *__restrict__ wE, int F_in, int F_out,
                                       float *__restrict__ dst) {
  const int64_t n1 = (int64_t)F_in * F_out;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < 4 * n1) {
    const int c = (int)(idx / n1);
    const int64_t r = idx % n1;
    const int i = (int)(r / F_out), o = (int)(r % F_out);
    const T *src = c == 0 ? a1 : c == 1 ? a2 : c == 2 ? b1 : b2;
    dst[idx] = to_f32(src[(size_t)o * F_in + i]);
  } else if (idx < 8 * n1) {
    const int64_t r = idx - 4 * n1;
    const int e = (int)(r / (2 * F_out)), e2 = (int)(r % (2 * F_out));
    dst[idx] = to_f32(wE[(size_t)e2 * (2 * F_in) + e]);
  }
}

__device__ __forceinline__ float gelu_exact(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752440f));
}

template <typename T>
__global__ void __launch_bounds__(kFzThreads)
d8_fourier_linear_kernel(const T *__restrict__ z, const float *__restrict__ W1,
                         const float *__restrict__ WEt, T *__restrict__ y, int64_t Tn, int F_in,
                         int F_out, int roundtrip_gelu, D8Tables tab) {
  __shared__ float Zs[kFzTT][kFzIC][9];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kFzTT;
  const int o = blockIdx.y * kFzOT + lane;
  const size_t n1 = (size_t)F_in * F_out;

  float acc[kFzTPT][8];
#pragma unroll
  for (int a = 0; a < kFzTPT; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;

  for (int i0 = 0; i0 < F_in; i0 += kFzIC) {
    __syncthreads();
    for (int p = threadIdx.x; p < kFzTT * kFzIC; p += kFzThreads) {
      const int tl = p / kFzIC, il = p % kFzIC;
      const int64_t t = t0 + tl;
      const int i = i0 + il;
      if (t < Tn && i < F_in) {
        float v[8];
        load_field<8, T>(z + ((size_t)t * F_in + i) * 8, v);
#pragma unroll
        for (int c = 0; c < 8; ++c) Zs[tl][il][c] = v[c];
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) Zs[tl][il][c] = 0.f;
      }
    }
    __syncthreads();
    if (o < F_out) {
      const int iend = min(kFzIC, F_in - i0);
      for (int il = 0; il < iend; ++il) {
        const int i = i0 + il;
        float w[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = __ldg(W1 + c * n1 + (size_t)i * F_out + o);
        // wE^T rows e = 2i + b, columns e' = 2o + b'
        const float2 e0 =
            __ldg(reinterpret_cast<const float2 *>(WEt + (size_t)(2 * i) * (2 * F_out) + 2 * o));
        const float2 e1 =
            __ldg(reinterpret_cast<const float2 *>(WEt + (size_t)(2 * i + 1) * (2 * F_out) + 2 * o));
#pragma unroll
        for (int a = 0; a < kFzTPT; ++a) {
          const float *zz = Zs[warp * kFzTPT + a][il];
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(w[c], zz[c], acc[a][c]);
#pragma unroll
          for (int ra = 0; ra < 2; ++ra) {
            const float zb0 = zz[4 + 2 * ra + 0], zb1 = zz[4 + 2 * ra + 1];
            acc[a][4 + 2 * ra + 0] = fmaf(e0.x, zb0, fmaf(e1.x, zb1, acc[a][4 + 2 * ra + 0]));
            acc[a][4 + 2 * ra + 1] = fmaf(e0.y, zb0, fmaf(e1.y, zb1, acc[a][4 + 2 * ra + 1]));
          }
        }
      }
    }
  }
  if (o >= F_out) return;
#pragma unroll
  for (int a = 0; a < kFzTPT; ++a) {
    const int64_t t = t0 + warp * kFzTPT + a;
    if (t >= Tn) continue;
    T *dst = y + ((size_t)t * F_out + o) * 8;
    if (roundtrip_gelu) {
      // regular slots x_g = sum_c Q[c][g] acc_c, GELU, back: z'_c = sum_g Q[c][g] GELU(x_g)
      float gx[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) s = fmaf(tab.q[c][g], acc[a][c], s);
        gx[g] = gelu_exact(s);
      }
      float zv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) s = fmaf(tab.q[c][g], gx[g], s);
        zv[c] = s;
      }
      store_field<8, T>(dst, zv);
    } else {
      store_field<8, T>(dst, acc[a]);
    }
  }
}

template <typename T>
int dispatch_linear(const T *z, const float *W1, const float *WEt, T *y, int64_t Tn, int F_in,
                    int F_out, int gelu, cudaStream_t s) {
  D8Tables tab;
  make_d8_tables(&tab);
  const int64_t gx = (Tn + kFzTT - 1) / kFzTT;
  if (gx > 0x7fffffffLL) return set_error(EQLIN_ERR_UNSUPPORTED, "T too large for the grid");
  dim3 grid((unsigned)gx, (unsigned)((F_out + kFzOT - 1) / kFzOT));
  d8_fourier_linear_kernel<T><<<grid, kFzThreads, 0, s>>>(z, W1, WEt, y, Tn, F_in, F_out, gelu, tab);
  return check_launch("d8 Fourier-domain linear");
}

// Sum of the S column-slice partial outputs of a wide layer (bf16, each
// [T][F_out][8]) in slice order, in fp32; with roundtrip_gelu the sum then goes
// through Q GELU(Q^T .).  One thread per (token, output field).
__global__ void d8_slice_sum_kernel(const __nv_bfloat16 *__restrict__ parts, int S, int64_t items,
                                    int roundtrip_gelu, D8Tables tab, __nv_bfloat16 *__restrict__ y) {
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    float z[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) z[c] = 0.f;
    for (int sl = 0; sl < S; ++sl) {
      const uint4 v = *reinterpret_cast<const uint4 *>(parts + ((size_t)sl * items + it) * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        z[2 * k] += __uint_as_float(w[k] << 16);
        z[2 * k + 1] += __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
    if (roundtrip_gelu) {
      float gx[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) a = fmaf(tab.q[c][g], z[c], a);
        gx[g] = gelu_exact(a);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float a = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) a = fmaf(tab.q[c][g], gx[g], a);
        z[c] = a;
      }
    }
    uint4 o;
    uint32_t *ow = &o.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 h = __floats2bfloat162_rn(z[2 * k], z[2 * k + 1]);
      ow[k] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(y + (size_t)it * 8) = o;
  }
}

}  // namespace

int launch_d8_slice_sum(const void *parts, int S, int64_t T, int F_out, int roundtrip_gelu, void *y,
                        cudaStream_t s) {
  D8Tables tab;
  make_d8_tables(&tab);
  const int64_t items = T * (int64_t)F_out;
  const int64_t want = (items + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  d8_slice_sum_kernel<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(parts), S, items,
                                              roundtrip_gelu, tab, static_cast<__nv_bfloat16 *>(y));
  return check_launch("d8 slice sum");
}

size_t d8_fourier_pack_bytes(int F_in, int F_out) {
  return 8 * (size_t)F_in * (size_t)F_out * sizeof(float);
}

int launch_d8_fourier_pack(const void *const w[5], int F_in, int F_out, int dtype, void *Wpack,
                           cudaStream_t s) {
  float *dst = static_cast<float *>(Wpack);
  const int64_t n = 8LL * F_in * F_out;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (dtype == EQLIN_F32)
    d8_fourier_pack_kernel<float><<<blocks, threads, 0, s>>>(
        (const float *)w[0], (const float *)w[1], (const float *)w[2], (const float *)w[3],
        (const float *)w[4], F_in, F_out, dst);
  else if (dtype == EQLIN_F16)
    d8_fourier_pack_kernel<__half><<<blocks, threads, 0, s>>>(
        (const __half *)w[0], (const __half *)w[1], (const __half *)w[2], (const __half *)w[3],
        (const __half *)w[4], F_in, F_out, dst);
  else
    d8_fourier_pack_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        (const __nv_bfloat16 *)w[0], (const __nv_bfloat16 *)w[1], (const __nv_bfloat16 *)w[2],
        (const __nv_bfloat16 *)w[3], (const __nv_bfloat16 *)w[4], F_in, F_out, dst);
  return check_launch("d8 Fourier-domain weight pack");
}

int launch_d8_fourier_linear(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                             int gelu, int dtype, cudaStream_t s) {
  const float *W1 = static_cast<const float *>(Wpack);
  const float *WEt = W1 + 4 * (size_t)F_in * F_out;
  if (dtype == EQLIN_F32)
    return dispatch_linear((const float *)z, W1, WEt, (float *)y, T, F_in, F_out, gelu, s);
  if (dtype == EQLIN_F16)
    return dispatch_linear((const __half *)z, W1, WEt, (__half *)y, T, F_in, F_out, gelu, s);
  return dispatch_linear((const __nv_bfloat16 *)z, W1, WEt, (__nv_bfloat16 *)y, T, F_in, F_out, gelu, s);
}

}  // namespace eqlin
