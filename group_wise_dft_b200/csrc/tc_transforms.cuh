// Device helpers shared by the tensor-core kernels: paired fp32 arithmetic,
// the forward real DFT of 8 group slots, and bf16 packing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace eqlin {

// Every transform works on two independent vectors at once (two fields, or
// two (token, field) items): each float2 lane of a value is one vector, and
// the arithmetic uses sm_100's paired fp32 instructions (add/mul/fma on
// float2), halving the instruction count of these ALU-bound steps.  Each
// paired operation rounds each lane exactly as the scalar one would.

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);   // a - b, one rounding
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 scl2(float2 a, float s) { return __fmul2_rn(a, make_float2(s, s)); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Cyclic C_8 half spectrum (real coordinates [Re X0, Re X1, Im X1, Re X2,
// Im X2, Re X3, Im X3, Re X4]) by a radix-2 split: the even bins are the
// 4-point DFT of x_h + x_{h+4}, the odd bins come from x_h - x_{h+4}.
__device__ __forceinline__ void fwd_cyclic8(const float2 (&x)[8], float2 (&z)[8]) {
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
__device__ __forceinline__ void unpack_f16x8_pair(const uint4 &a, const uint4 &b, float2 (&f)[8]) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 fa = __half22float2(*reinterpret_cast<const __half2 *>(&wa[k]));
    const float2 fb = __half22float2(*reinterpret_cast<const __half2 *>(&wb[k]));
    f[2 * k] = make_float2(fa.x, fb.x);
    f[2 * k + 1] = make_float2(fa.y, fb.y);
  }
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
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
