// Device helpers shared by the tensor-core kernels: paired fp32 arithmetic,
// the forward real DFT of 8 group slots, and bf16 packing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

namespace eqlin {

// Every transform works on two independent vectors at once (two fields, or
// two (token, field) items): each float2 lane of a value is one vector, and
// the arithmetic uses sm_100's paired fp32 instructions (add/mul/fma on
// float2), halving the instruction count of these ALU-bound steps.  Each
// paired operation rounds each lane exactly as the scalar one would.

// (Host builds, used only by the CPU tests of these transforms, take the
// scalar operations, which round the same way.)
__host__ __device__ __forceinline__ float2 add2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
  return __fadd2_rn(a, b);
#else
  return make_float2(a.x + b.x, a.y + b.y);
#endif
}
__host__ __device__ __forceinline__ float2 sub2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);   // a - b, one rounding
#else
  return make_float2(a.x - b.x, a.y - b.y);
#endif
}
__host__ __device__ __forceinline__ float2 mul2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
  return __fmul2_rn(a, b);
#else
  return make_float2(a.x * b.x, a.y * b.y);
#endif
}
__host__ __device__ __forceinline__ float2 scl2(float2 a, float s) { return mul2(a, make_float2(s, s)); }
__host__ __device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
#ifdef __CUDA_ARCH__
  return __ffma2_rn(a, b, c);
#else
  return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}

// Cyclic C_8 half spectrum (real coordinates [Re X0, Re X1, Im X1, Re X2,
// Im X2, Re X3, Im X3, Re X4]) by a radix-2 split: the even bins are the
// 4-point DFT of x_h + x_{h+4}, the odd bins come from x_h - x_{h+4}.
__host__ __device__ __forceinline__ void fwd_cyclic8(const float2 (&x)[8], float2 (&z)[8]) {
  const float r = 0.70710678118654752f;
  const float2 e0 = add2(x[0], x[4]), e1 = add2(x[1], x[5]), e2 = add2(x[2], x[6]),
               e3 = add2(x[3], x[7]);
  const float2 d0 = sub2(x[0], x[4]), d1 = sub2(x[1], x[5]), d2 = sub2(x[2], x[6]),
               d3 = sub2(x[3], x[7]);
  const float2 s02 = add2(e0, e2), s13 = add2(e1, e3);
  const float2 p = scl2(sub2(d1, d3), r), q = scl2(add2(d1, d3), r);
  z[0] = add2(s02, s13);
  z[7] = sub2(s02, s13);
  z[3] = sub2(e0, e2);
  z[4] = sub2(e3, e1);
  z[1] = add2(d0, p);
  z[2] = sub2(scl2(d2, -1.0f), q);
  z[5] = sub2(d0, p);
  z[6] = sub2(d2, q);
}

// Inverse: y_g = Y0 + (-1)^g Y4 + sum_{k=1..3} Re(Y'_k e^{2 pi i g k / 8}); the
// complex bins arrive already doubled (Y' = 2Y, folded into the weights) and
// the 1/8 is in the weights too.  Even part E (period 4) + odd part O
// (O_{g+4} = -O_g).
__host__ __device__ __forceinline__ void inv_cyclic8(const float2 (&z)[8], float2 (&y)[8]) {
  const float r = 0.70710678118654752f;
  const float2 y0 = z[0], y4 = z[7], a = z[1], b = z[2], c2r = z[3], c2i = z[4], c = z[5],
               d = z[6];
  const float2 p = add2(y0, y4), m = sub2(y0, y4);
  const float2 E0 = add2(p, c2r), E1 = sub2(m, c2i), E2 = sub2(p, c2r), E3 = add2(m, c2i);
  const float2 bd = add2(b, d);
  const float2 O0 = add2(a, c), O1 = scl2(sub2(sub2(a, c), bd), r), O2 = sub2(d, b),
               O3 = scl2(sub2(sub2(c, a), bd), r);
  y[0] = add2(E0, O0);
  y[1] = add2(E1, O1);
  y[2] = add2(E2, O2);
  y[3] = add2(E3, O3);
  y[4] = sub2(E0, O0);
  y[5] = sub2(E1, O1);
  y[6] = sub2(E2, O2);
  y[7] = sub2(E3, O3);
}

// cos(m pi / 8), m taken modulo 16 (sin(m pi / 8) = cos((m - 4) pi / 8)).
__host__ __device__ constexpr float cos_pi8(int m) {
  constexpr float c1 = 0.92387953251128674f;   // cos(pi/8)
  constexpr float c2 = 0.70710678118654752f;   // cos(pi/4)
  constexpr float c3 = 0.38268343236508977f;   // cos(3pi/8)
  switch (m & 15) {
    case 0: return 1.0f;
    case 1: return c1;
    case 2: return c2;
    case 3: return c3;
    case 4: return 0.0f;
    case 5: return -c3;
    case 6: return -c2;
    case 7: return -c1;
    case 8: return -1.0f;
    case 9: return -c1;
    case 10: return -c2;
    case 11: return -c3;
    case 12: return 0.0f;
    case 13: return c3;
    case 14: return c2;
    default: return c1;
  }
}
__host__ __device__ constexpr float sin_pi8(int m) { return cos_pi8(m - 4); }

// Negacyclic C_8 spectrum (the product modulo z^8 + 1 diagonalises at the odd
// 16th roots of unity): D_b = sum_h d_h e^{-i pi h (2b+1) / 8}, b = 0..3, as
// real coordinates [Re D0, Im D0, .., Re D3, Im D3]; D_{7-b} = conj(D_b) for
// real d, so these four bins carry it all.
__host__ __device__ __forceinline__ void fwd_negacyclic8(const float2 (&x)[8], float2 (&z)[8]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float2 re = make_float2(0.0f, 0.0f), im = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float c = cos_pi8(h * (2 * b + 1)), sn = sin_pi8(h * (2 * b + 1));
      if (c != 0.0f) re = fma2(x[h], make_float2(c, c), re);
      if (sn != 0.0f) im = fma2(x[h], make_float2(-sn, -sn), im);
    }
    z[2 * b] = re;
    z[2 * b + 1] = im;
  }
}

// Inverse: y_g = sum_{b=0..3} Re(Y_b e^{i pi g (2b+1) / 8}); the 2/8 of the
// one-sided inverse is in the weights.
__host__ __device__ __forceinline__ void inv_negacyclic8(const float2 (&z)[8], float2 (&y)[8]) {
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    float2 v = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float c = cos_pi8(g * (2 * b + 1)), sn = sin_pi8(g * (2 * b + 1));
      if (c != 0.0f) v = fma2(z[2 * b], make_float2(c, c), v);
      if (sn != 0.0f) v = fma2(z[2 * b + 1], make_float2(-sn, -sn), v);
    }
    y[g] = v;
  }
}

// D8 change of basis Q (rows A1, A2, B1, B2, E00, E01, E10, E11) through the
// sums u_j = x(r^j) + x(r^j s) and differences v_j = x(r^j) - x(r^j s).
__host__ __device__ __forceinline__ void fwd_d8(const float2 (&x)[8], float2 (&z)[8]) {
  const float is8 = 0.35355339059327376f;  // 1/sqrt(8)
  const float2 u0 = add2(x[0], x[4]), u1 = add2(x[1], x[5]), u2 = add2(x[2], x[6]),
               u3 = add2(x[3], x[7]);
  const float2 v0 = sub2(x[0], x[4]), v1 = sub2(x[1], x[5]), v2 = sub2(x[2], x[6]),
               v3 = sub2(x[3], x[7]);
  const float2 u02 = add2(u0, u2), u13 = add2(u1, u3), v02 = add2(v0, v2), v13 = add2(v1, v3);
  z[0] = scl2(add2(u02, u13), is8);
  z[1] = scl2(add2(v02, v13), is8);
  z[2] = scl2(sub2(u02, u13), is8);
  z[3] = scl2(sub2(v02, v13), is8);
  z[4] = scl2(sub2(u0, u2), 0.5f);
  z[5] = scl2(sub2(v3, v1), 0.5f);
  z[6] = scl2(sub2(u1, u3), 0.5f);
  z[7] = scl2(sub2(v0, v2), 0.5f);
}

// x = Q^T z.
__host__ __device__ __forceinline__ void inv_d8(const float2 (&z)[8], float2 (&x)[8]) {
  const float r = 0.70710678118654752f;
  const float2 ap = scl2(add2(z[0], z[2]), r), am = scl2(sub2(z[0], z[2]), r);
  const float2 bp = scl2(add2(z[1], z[3]), r), bm = scl2(sub2(z[1], z[3]), r);
  const float2 U0 = add2(ap, z[4]), U1 = add2(am, z[6]), U2 = sub2(ap, z[4]), U3 = sub2(am, z[6]);
  const float2 V0 = add2(bp, z[7]), V1 = sub2(bm, z[5]), V2 = sub2(bp, z[7]), V3 = add2(bm, z[5]);
  x[0] = scl2(add2(U0, V0), 0.5f);
  x[1] = scl2(add2(U1, V1), 0.5f);
  x[2] = scl2(add2(U2, V2), 0.5f);
  x[3] = scl2(add2(U3, V3), 0.5f);
  x[4] = scl2(sub2(U0, V0), 0.5f);
  x[5] = scl2(sub2(U1, V1), 0.5f);
  x[6] = scl2(sub2(U2, V2), 0.5f);
  x[7] = scl2(sub2(U3, V3), 0.5f);
}

// GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)).  erf is taken from
// Abramowitz & Stegun, Handbook of Mathematical Functions, eq. 7.1.28
// (Hastings): for x >= 0, erf(x) = 1 - (1 + a1 x + ... + a6 x^6)^-16 with
// |error| <= 3e-7 (about 2e-6 after fp32 rounding); odd symmetry covers
// x < 0.  With r = (1 + ...)^-16 at x = |v| / sqrt 2 and h = v r / 2:
// GELU(v) = v - h for v >= 0 and h for v < 0.  One reciprocal per value,
// no exponential.
__host__ __device__ __forceinline__ float2 gelu_erf2(float2 v) {
  const float2 x = scl2(make_float2(fabsf(v.x), fabsf(v.y)), 0.70710678118654752f);
  float2 p = make_float2(0.0000430638f, 0.0000430638f);
  p = fma2(p, x, make_float2(0.0002765672f, 0.0002765672f));
  p = fma2(p, x, make_float2(0.0001520143f, 0.0001520143f));
  p = fma2(p, x, make_float2(0.0092705272f, 0.0092705272f));
  p = fma2(p, x, make_float2(0.0422820123f, 0.0422820123f));
  p = fma2(p, x, make_float2(0.0705230784f, 0.0705230784f));
  p = fma2(p, x, make_float2(1.0f, 1.0f));
  p = mul2(p, p);   // ^2
  p = mul2(p, p);   // ^4
  p = mul2(p, p);   // ^8
  p = mul2(p, p);   // ^16
#ifdef __CUDA_ARCH__
  const float2 q = make_float2(__fdividef(1.0f, p.x), __fdividef(1.0f, p.y));
#else
  const float2 q = make_float2(1.0f / p.x, 1.0f / p.y);
#endif
  const float2 h = mul2(scl2(v, 0.5f), q);
  return make_float2(v.x >= 0.0f ? v.x - h.x : h.x, v.y >= 0.0f ? v.y - h.y : h.y);
}

// GELU through the tanh form of Hendrycks and Gimpel (Gaussian Error Linear
// Units, 2016): GELU(v) ~ 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))).
// Its largest deviation from the exact-erf GELU is 4.8e-4 (at |v| = 2.7; a
// CPU test pins it), and the hardware tanh (tanh.approx.f32, relative error
// about 2^-11) adds at most 0.5 |v| 2^-11 more; both stay far below the
// rounding of a bf16 output (2^-9 relative).  Five paired operations and one
// tanh per value, against the erf form's sixteen and a reciprocal: the D8
// epilogue, which applies it to every output, is the busiest role of that
// layer's kernel.
__host__ __device__ __forceinline__ float tanh_fast(float u) {
#ifdef __CUDA_ARCH__
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  return t;
#else
  return tanhf(u);
#endif
}
__host__ __device__ __forceinline__ float2 gelu_tanh2(float2 v) {
  const float k0 = 0.79788456080286536f;          // sqrt(2 / pi)
  const float k1 = 0.79788456080286536f * 0.044715f;
  const float2 v2 = mul2(v, v);
  const float2 u = mul2(v, fma2(v2, make_float2(k1, k1), make_float2(k0, k0)));
  const float2 t = make_float2(tanh_fast(u.x), tanh_fast(u.y));
  const float2 h = scl2(v, 0.5f);
  return fma2(h, t, h);
}

// p4 (C_4) on the fused kernel: a 16-byte chunk holds two C_4 fields (a
// "super-field" of 8 slots).  The 4-point DFT has entries 0, +-1, +-i, so
// both transforms are additions.  Coordinates per C_4 field: [Re X0, Re X1,
// Im X1, Re X2], X_1 = x0 - x2 + i (x3 - x1); z[0..3] for the super-field's
// first field, z[4..7] for its second.
__host__ __device__ __forceinline__ void fwd_cyclic4x2(const float2 (&x)[8], float2 (&z)[8]) {
#pragma unroll
  for (int f = 0; f < 2; ++f) {
    const float2 *v = x + 4 * f;
    const float2 e = add2(v[0], v[2]), o = add2(v[1], v[3]);
    z[4 * f + 0] = add2(e, o);
    z[4 * f + 1] = sub2(v[0], v[2]);
    z[4 * f + 2] = sub2(v[3], v[1]);
    z[4 * f + 3] = sub2(e, o);
  }
}

// Inverse per C_4 field with the complex bin already doubled and the 1/4 in
// the weights: y_g = Y0 + (-1)^g Y2 + Re(Y'_1 i^g).
__host__ __device__ __forceinline__ void inv_cyclic4x2(const float2 (&z)[8], float2 (&y)[8]) {
#pragma unroll
  for (int f = 0; f < 2; ++f) {
    const float2 *c = z + 4 * f;
    const float2 p = add2(c[0], c[3]), m = sub2(c[0], c[3]);
    y[4 * f + 0] = add2(p, c[1]);
    y[4 * f + 1] = sub2(m, c[2]);
    y[4 * f + 2] = sub2(p, c[1]);
    y[4 * f + 3] = add2(m, c[2]);
  }
}

// Two bf16x8 vectors (one 16-byte chunk each) to 8 float2 (a in .x, b in .y).
__device__ __forceinline__ void unpack_bf16x8_pair(const uint4 &a, const uint4 &b, float2 (&f)[8]) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = make_float2(__uint_as_float(wa[k] << 16), __uint_as_float(wb[k] << 16));
    f[2 * k + 1] = make_float2(__uint_as_float(wa[k] & 0xFFFF0000u), __uint_as_float(wb[k] & 0xFFFF0000u));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// The same for fp16 data: two fp16x8 vectors to 8 float2, and a float pair to
// fp16x2 (round to nearest).
__host__ __device__ __forceinline__ void unpack_f16x8_pair(const uint4 &a, const uint4 &b, float2 (&f)[8]) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 fa = __half22float2(*reinterpret_cast<const __half2 *>(&wa[k]));
    const float2 fb = __half22float2(*reinterpret_cast<const __half2 *>(&wb[k]));
    f[2 * k] = make_float2(fa.x, fb.x);
    f[2 * k + 1] = make_float2(fa.y, fb.y);
  }
}

__host__ __device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// I/O and operand type of the tensor-core kernels: bf16 (H = false) or fp16.
template <bool H>
__device__ __forceinline__ void unpack_x8_pair(const uint4 &a, const uint4 &b, float2 (&f)[8]) {
  if (H)
    unpack_f16x8_pair(a, b, f);
  else
    unpack_bf16x8_pair(a, b, f);
}
template <bool H>
__device__ __forceinline__ uint32_t pack_x2(float lo, float hi) {
  return H ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

}  // namespace eqlin
