// Weight-side arithmetic of the tensor-core path's packing: where a layer's
// 8-slot weight comes from (plain, adjoint, the two folds of a 16-slot
// weight), and the value of each entry of the per-field spectral block matrix.
// Host-and-device so that the CPU tests can run it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stddef.h>

namespace eqlin {

// Modes of the fused kernel: cyclic C_8, the D8 Fourier-domain layer, and the
// negacyclic C_8 layer (the odd half of a C_16 layer).
constexpr int kModeCyclic8 = 0;
constexpr int kModeD8 = 1;
constexpr int kModeNegacyclic8 = 2;
// p4: C_4 fields in pairs (super-fields of 8 slots); F_in counts super-fields,
// F_out C_4 fields.
constexpr int kModeCyclic4 = 3;

// D8 weight blocks: w[0..3] [F_out][ld1] (the layer's F_in columns first),
// w[4] [2 F_out][ldE]; ld1 = F_in and ldE = 2 F_in unless the layer is a
// column slice of wider blocks.
struct D8Blocks {
  const __nv_bfloat16 *w[5];
  int ld1 = 0, ldE = 0;
};

// Value of the spectral block matrix: output coordinate cout of field o from
// input coordinate cin of field i (cyclic coordinates as in fwd_cyclic8, with
// the complex bins doubled for the one-sided inverse; D8 coordinates A1, A2,
// B1, B2, E00, E01, E10, E11).
// Where the 8-slot weight V[o][i][m] of a cyclic or negacyclic layer comes from:
constexpr int kWsrcPlain = 0;      // W[o][i][m], W stored [F_out][F_in][8]
constexpr int kWsrcAdjoint = 1;    // W[i][o][(-m) mod 8], W stored [F_in][F_out][8] (backward data pass)
constexpr int kWsrcFoldEven = 2;   // (W[o][i][m] + W[o][i][m+8]) / 2, W stored [F_out][F_in][16]
constexpr int kWsrcFoldOdd = 3;    // (W[o][i][m] - W[o][i][m+8]) / 2, W stored [F_out][F_in][16]
constexpr int kWsrcFoldEvenAdj = 4;   // the two folds of the adjoint 16-slot weight
constexpr int kWsrcFoldOddAdj = 5;    // V[o][i][m] = W[i][o][(-m) mod 16], W stored [F_in][F_out][16]
// (the folds are the even and odd halves of a C_16 weight, each with the 1/2 of
// y_g = (Y_e + Y_o)/2, y_{g+8} = (Y_e - Y_o)/2 folded in)
// Element idx of a weight array of type WT (0: bf16, 1: fp16, 2: fp32), widened to double.
template <int WT>
__host__ __device__ __forceinline__ double ld_w(const void *W, size_t idx) {
  return WT == 2 ? (double)static_cast<const float *>(W)[idx]
       : WT == 1 ? (double)__half2float(static_cast<const __half *>(W)[idx])
                 : (double)__bfloat162float(static_cast<const __nv_bfloat16 *>(W)[idx]);
}

template <int H>
__host__ __device__ double cyclic_weight(const void *Wc, int F_in, int F_out, int wsrc, int o, int i, int m) {
  if (wsrc == kWsrcPlain) return ld_w<H>(Wc, ((size_t)o * F_in + i) * 8 + m);
  if (wsrc == kWsrcAdjoint) return ld_w<H>(Wc, ((size_t)i * F_out + o) * 8 + (8 - m) % 8);
  const bool adj = wsrc >= kWsrcFoldEvenAdj;
  auto v = [&](int mm) -> double {
    return ld_w<H>(Wc, adj ? ((size_t)i * F_out + o) * 16 + (16 - mm) % 16 : ((size_t)o * F_in + i) * 16 + mm);
  };
  const bool even = wsrc == kWsrcFoldEven || wsrc == kWsrcFoldEvenAdj;
  return 0.5 * (even ? v(m) + v(m + 8) : v(m) - v(m + 8));
}

// The 4-slot weight V[o][i][m] of a C_4 layer (W stored [F_out][F_in][4]), or
// for the backward data pass W[i][o][(-m) mod 4] (W stored [F_in][F_out][4]).
template <int H>
__host__ __device__ double c4_weight(const void *Wc, int F_in, int F_out, int adjoint, int o, int i, int m) {
  return adjoint ? ld_w<H>(Wc, ((size_t)i * F_out + o) * 4 + (4 - m) % 4)
                 : ld_w<H>(Wc, ((size_t)o * F_in + i) * 4 + m);
}

// C_4 block entry: coordinates [Re 0, Re 1, Im 1, Re 2], W_k = (1/4) sum_m V_m
// e^{-2 pi i m k / 4} (quarter-turn twiddles, exact), the complex bin doubled
// for the one-sided inverse.  F_in, F_out count C_4 fields here.
template <int H>
__host__ __device__ double c4_block_value(const void *Wc, int F_in, int F_out, int adjoint, int cout, int o,
                                          int cin, int i) {
  const int bin = cout == 0 ? 0 : (cout == 3 ? 2 : 1);
  const double cq[4] = {1.0, 0.0, -1.0, 0.0}, sq[4] = {0.0, 1.0, 0.0, -1.0};
  double re = 0.0, im = 0.0;
  for (int m = 0; m < 4; ++m) {
    const double w = c4_weight<H>(Wc, F_in, F_out, adjoint, o, i, m);
    re += w * cq[(m * bin) & 3];
    im -= w * sq[(m * bin) & 3];
  }
  re *= 0.25;
  im *= 0.25;
  if (bin != 1) return re;
  const bool out_re = cout == 1, in_re = cin == 1;
  return 2.0 * (out_re ? (in_re ? re : -im) : (in_re ? im : re));
}

template <int MODE, int H>
__host__ __device__ double block_value(const void *Wc, const D8Blocks &d8, int F_in, int F_out,
                              int wsrc, int cout, int o, int cin, int i) {
  if (MODE == kModeNegacyclic8) {
    // coordinates [Re D0, Im D0, .., Re D3, Im D3]; bin b weight (2/8) sum_m V_m e^{-i pi m (2b+1)/8}
    const int b = cout >> 1;
    double re = 0.0, im = 0.0;
    for (int m = 0; m < 8; ++m) {
      const double w = cyclic_weight<H>(Wc, F_in, F_out, wsrc, o, i, m);
      const double ang = M_PI * (double)((m * (2 * b + 1)) % 16) / 8.0;
      re += w * cos(ang);
      im -= w * sin(ang);
    }
    re *= 2.0 / 8.0;
    im *= 2.0 / 8.0;
    const bool out_re = (cout & 1) == 0, in_re = (cin & 1) == 0;
    return out_re ? (in_re ? re : -im) : (in_re ? im : re);
  }
  if (MODE == kModeCyclic8) {
    const int bin = cout == 0 ? 0 : (cout == 7 ? 4 : (cout + 1) / 2);
    double re = 0.0, im = 0.0;
    for (int m = 0; m < 8; ++m) {
      const double w = cyclic_weight<H>(Wc, F_in, F_out, wsrc, o, i, m);
      const double ang = 2.0 * M_PI * (double)((m * bin) % 8) / 8.0;
      re += w * cos(ang);
      im -= w * sin(ang);
    }
    re /= 8.0;
    im /= 8.0;
    if (bin == 0 || bin == 4) return re;
    const bool out_re = (cout & 1) == 1, in_re = (cin & 1) == 1;
    // [Yr; Yi] = [[Wr, -Wi], [Wi, Wr]] [Xr; Xi]
    return 2.0 * (out_re ? (in_re ? re : -im) : (in_re ? im : re));
  }
  if (cout < 4) return (double)__bfloat162float(d8.w[cout][(size_t)o * d8.ld1 + i]);
  const int bo = (cout - 4) & 1, bi = (cin - 4) & 1;
  return (double)__bfloat162float(d8.w[4][(size_t)(2 * o + bo) * d8.ldE + 2 * i + bi]);
}

}  // namespace eqlin
