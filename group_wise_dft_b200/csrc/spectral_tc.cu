// Fused tcgen05 tensor-core path for layers with 8 group slots per field:
// cyclic C_8 EQ-Linear (Flash EQ-Linear, Methodology > Algorithmic Approach:
// real DFT along the group axis, per-bin complex products, inverse DFT) and
// the D8 Fourier-domain linear layer (Quick ViTs review, Key design 2:
// change of basis to irreps, Schur blocks with E shared over its two row
// coordinates, back-transform, GELU in the regular domain).
//
// One kernel does the whole layer; the spectra never leave the SM.
//
//   CTA pair (cluster of 2, tcgen05 cta_group::2, instruction M = 128):
//   each CTA owns 64 token rows of a 128-token tile.  Per CTA:
//     x producer warp   TMA-loads x in boxes of 64 tokens x 8 fields (SW128)
//     DFT warps (4)     8-point transform of every field, written as the
//                       K-major bf16 A operand: 8 coordinate blocks x Fin
//                       (the whole tile's spectrum stays resident: Fin KB)
//     B producer warp   TMA-loads pre-packed weight panels (its half of N)
//     MMA thread        (leader CTA) per output chunk of up to 64 fields,
//                       per job: K-steps of 16 into a double-buffered TMEM
//                       accumulator (4 * chunk columns per buffer)
//     epilogue warps(4) TMEM -> registers, inverse 8-point transform,
//                       optional GELU, bf16 stores of y
//
// "Jobs" are the per-bin (cyclic) or per-irrep (D8) block products:
//   real job   : one coordinate block, K = Fin,  N = chunk      (bins 0, 4;
//                A1, A2, B1, B2)
//   paired job : two adjacent blocks,  K = 2Fin, N = 2*chunk    (complex bins
//                1..3 as [[Re, Im],[-Im, Re]] real blocks; D8 E with one B
//                panel applied to both row coordinates a = 0, 1)
//
// Every wait on an mbarrier is bounded: on timeout the kernel records a code
// in g_fault_word, stops issuing work, lets copies in flight land, frees its
// TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "eqlin_internal.cuh"
#include "tc_primitives.cuh"

namespace eqlin {

__device__ unsigned int g_fault_word = 0;

int read_device_fault(int reset) {
  unsigned int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return -(int)e;
  e = cudaMemcpyFromSymbol(&v, g_fault_word, sizeof v);
  if (e != cudaSuccess) return -(int)e;
  if (reset && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_fault_word, &z, sizeof z);
    if (e != cudaSuccess) return -(int)e;
  }
  return (int)v;
}

namespace {

constexpr int kModeCyclic8 = 0;
constexpr int kModeD8 = 1;

constexpr int kThreads = 384;
constexpr int kWarpX = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpB = 2;
constexpr int kDftWarp0 = 4;
constexpr int kNumDftWarps = 4;
constexpr int kEpiWarp0 = 8;
constexpr int kNumEpiWarps = 4;

constexpr int kRowsPerCta = 64;
constexpr int kTileTokens = 2 * kRowsPerCta;
constexpr int kXStages = 4;
constexpr int kXStageBytes = kRowsPerCta * 128;  // 64 tokens x 8 fields x 8 slots x bf16
constexpr int kBStages = 8;
constexpr int kBStageBytes = 4096;
constexpr int kCoMax = 64;     // output fields per chunk
constexpr int kMaxFin = 160;   // A operand = Fin KB of shared memory
constexpr int kKPiece = 32;    // K elements per B stage
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccBufCols = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kNumJobs = 5;
constexpr int kNumBars = 31;

struct JobDesc {
  int ncoord;     // 1 = real job, 2 = paired job
  int ntarget;    // A/D targets sharing the B panel
  int acoord[2];  // first A coordinate block of each target
  int dgroup[2];  // first D column group (units of chunk/2 columns) of each target
};

__host__ __device__ inline JobDesc job_desc(int mode, int j) {
  if (mode == kModeCyclic8) {
    // coordinates: 0 = Re X0, 1/2 = X1, 3/4 = X2, 5/6 = X3, 7 = Re X4
    switch (j) {
      case 0: return {1, 1, {0, 0}, {0, 0}};
      case 1: return {1, 1, {7, 0}, {1, 0}};
      case 2: return {2, 1, {1, 0}, {2, 0}};
      case 3: return {2, 1, {3, 0}, {4, 0}};
      default: return {2, 1, {5, 0}, {6, 0}};
    }
  }
  // D8: 0 A1, 1 A2, 2 B1, 3 B2, 4/5 = E row a=0 (b=0,1), 6/7 = E row a=1
  switch (j) {
    case 0: return {1, 1, {0, 0}, {0, 0}};
    case 1: return {1, 1, {1, 0}, {1, 0}};
    case 2: return {1, 1, {2, 0}, {2, 0}};
    case 3: return {1, 1, {3, 0}, {3, 0}};
    default: return {2, 2, {4, 6}, {4, 6}};
  }
}

// Coordinate held by TMEM column group k (k = 0..7) of an accumulator buffer.
__host__ __device__ inline int group_coord(int mode, int k) {
  if (mode == kModeCyclic8) {
    const int map[8] = {0, 7, 1, 2, 3, 4, 5, 6};
    return map[k];
  }
  return k;
}

__host__ __device__ inline int chunk_fields(int F_out, int c) {
  const int r = F_out - c * kCoMax;
  return r < kCoMax ? r : kCoMax;
}
__host__ __device__ inline int num_chunks(int F_out) { return (F_out + kCoMax - 1) / kCoMax; }
__host__ __device__ inline int job_rows(const JobDesc &jd, int co) {
  return jd.ncoord == 1 ? co / 2 : co;
}
__host__ __device__ inline int job_pieces(const JobDesc &jd, int F_in) {
  return jd.ncoord * F_in / kKPiece;
}

// Offset, in 16-byte rows, of the packed panels of (chunk c, job j).  Within a
// job the panels are ordered (piece p, CTA half h), each 4*R rows laid out
// [K-chunk 0..3][R output rows][8 bf16] -- the shared-memory image of one B
// stage.  Called with (c = nchunks, j = 0) it returns the total row count.
__host__ __device__ inline int64_t b_job_base(int mode, int F_in, int F_out, int c, int j) {
  int64_t off = 0;
  const int nch = num_chunks(F_out);
  for (int cc = 0; cc < nch; ++cc) {
    const int co = chunk_fields(F_out, cc);
    for (int jj = 0; jj < kNumJobs; ++jj) {
      if (cc == c && jj == j) return off;
      const JobDesc jd = job_desc(mode, jj);
      off += (int64_t)job_pieces(jd, F_in) * 2 * 4 * job_rows(jd, co);
    }
  }
  return off;
}

size_t smem_bytes_for(int F_in) {
  return 1024 + (size_t)F_in * 1024 + kXStages * kXStageBytes + kBStages * kBStageBytes + 256;
}

// ---------------------------------------------------------------- transforms
// Cyclic C_8 half spectrum (real coordinates [Re X0, Re X1, Im X1, Re X2,
// Im X2, Re X3, Im X3, Re X4]) by a radix-2 split: the even bins are the
// 4-point DFT of x_h + x_{h+4}, the odd bins come from x_h - x_{h+4}.
__device__ __forceinline__ void fwd_cyclic8(const float (&x)[8], float (&z)[8]) {
  const float r = 0.70710678118654752f;
  const float e0 = x[0] + x[4], e1 = x[1] + x[5], e2 = x[2] + x[6], e3 = x[3] + x[7];
  const float d0 = x[0] - x[4], d1 = x[1] - x[5], d2 = x[2] - x[6], d3 = x[3] - x[7];
  const float s02 = e0 + e2, s13 = e1 + e3;
  const float p = (d1 - d3) * r, q = (d1 + d3) * r;
  z[0] = s02 + s13;
  z[7] = s02 - s13;
  z[3] = e0 - e2;
  z[4] = e3 - e1;
  z[1] = d0 + p;
  z[2] = -d2 - q;
  z[5] = d0 - p;
  z[6] = d2 - q;
}

// Inverse: y_g = Y0 + (-1)^g Y4 + sum_{k=1..3} Re(Y'_k e^{2 pi i g k / 8}); the
// complex bins arrive already doubled (Y' = 2Y, folded into the weights) and
// the 1/8 is in the weights too.  Even part E (period 4) + odd part O
// (O_{g+4} = -O_g).
__device__ __forceinline__ void inv_cyclic8(const float (&z)[8], float (&y)[8]) {
  const float r = 0.70710678118654752f;
  const float y0 = z[0], y4 = z[7], a = z[1], b = z[2], c2r = z[3], c2i = z[4], c = z[5], d = z[6];
  const float p = y0 + y4, m = y0 - y4;
  const float E0 = p + c2r, E1 = m - c2i, E2 = p - c2r, E3 = m + c2i;
  const float O0 = a + c, O1 = (a - b - c - d) * r, O2 = d - b, O3 = (c - a - b - d) * r;
  y[0] = E0 + O0;
  y[1] = E1 + O1;
  y[2] = E2 + O2;
  y[3] = E3 + O3;
  y[4] = E0 - O0;
  y[5] = E1 - O1;
  y[6] = E2 - O2;
  y[7] = E3 - O3;
}

// D8 change of basis Q (rows A1, A2, B1, B2, E00, E01, E10, E11) through the
// sums u_j = x(r^j) + x(r^j s) and differences v_j = x(r^j) - x(r^j s).
__device__ __forceinline__ void fwd_d8(const float (&x)[8], float (&z)[8]) {
  const float is8 = 0.35355339059327376f;  // 1/sqrt(8)
  const float u0 = x[0] + x[4], u1 = x[1] + x[5], u2 = x[2] + x[6], u3 = x[3] + x[7];
  const float v0 = x[0] - x[4], v1 = x[1] - x[5], v2 = x[2] - x[6], v3 = x[3] - x[7];
  z[0] = (u0 + u1 + u2 + u3) * is8;
  z[1] = (v0 + v1 + v2 + v3) * is8;
  z[2] = (u0 - u1 + u2 - u3) * is8;
  z[3] = (v0 - v1 + v2 - v3) * is8;
  z[4] = (u0 - u2) * 0.5f;
  z[5] = (v3 - v1) * 0.5f;
  z[6] = (u1 - u3) * 0.5f;
  z[7] = (v0 - v2) * 0.5f;
}

// x = Q^T z.
__device__ __forceinline__ void inv_d8(const float (&z)[8], float (&x)[8]) {
  const float r = 0.70710678118654752f;
  const float ap = (z[0] + z[2]) * r, am = (z[0] - z[2]) * r;
  const float bp = (z[1] + z[3]) * r, bm = (z[1] - z[3]) * r;
  const float U0 = ap + z[4], U1 = am + z[6], U2 = ap - z[4], U3 = am - z[6];
  const float V0 = bp + z[7], V1 = bm - z[5], V2 = bp - z[7], V3 = bm + z[5];
  x[0] = 0.5f * (U0 + V0);
  x[1] = 0.5f * (U1 + V1);
  x[2] = 0.5f * (U2 + V2);
  x[3] = 0.5f * (U3 + V3);
  x[4] = 0.5f * (U0 - V0);
  x[5] = 0.5f * (U1 - V1);
  x[6] = 0.5f * (U2 - V2);
  x[7] = 0.5f * (U3 - V3);
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------- kernel

struct TcArgs {
  int64_t T;
  int F_in;
  int F_out;
  int ntiles;
  int gelu;
  __nv_bfloat16 *y;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    spectral8_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_b16,
                        const __grid_constant__ CUtensorMap map_b32,
                        const __grid_constant__ CUtensorMap map_b64, const TcArgs args) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);

  const int F_in = args.F_in;
  const int F_out = args.F_out;
  const int nchunks = num_chunks(F_out);
  const int kcs = F_in / 8;  // K-chunks (8 elements) per coordinate block

  const uint32_t sA = base;
  const uint32_t sX = sA + (uint32_t)F_in * 1024u;
  const uint32_t sB = sX + kXStages * kXStageBytes;
  const uint32_t sBar = sB + kBStages * kBStageBytes;
  auto bar_x_full = [&](int i) { return sBar + 8u * i; };
  auto bar_x_empty = [&](int i) { return sBar + 8u * (4 + i); };
  auto bar_b_full = [&](int i) { return sBar + 8u * (8 + i); };
  auto bar_b_empty = [&](int i) { return sBar + 8u * (16 + i); };
  auto bar_acc_full = [&](int i) { return sBar + 8u * (24 + i); };
  auto bar_acc_empty = [&](int i) { return sBar + 8u * (26 + i); };
  const uint32_t bar_a_full = sBar + 8u * 28;
  const uint32_t bar_a_empty = sBar + 8u * 29;
  const uint32_t tmem_slot = sBar + 8u * 30;
  volatile uint32_t *tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t *>(gbase + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  unsigned int *fault = &g_fault_word;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) {
      mbar_init(bar_x_full(i), 1);
      mbar_init(bar_x_empty(i), 2);  // the two warps of the consuming DFT group
    }
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(bar_b_full(i), 1);
      mbar_init(bar_b_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc_full(i), 1);
      mbar_init(bar_acc_empty(i), 2 * kNumEpiWarps);
    }
    mbar_init(bar_a_full, 2 * kNumDftWarps);
    mbar_init(bar_a_empty, 1);
    fence_mbarrier_init_cluster();
  }
  if (warp == kWarpMma) tmem_alloc_pair(tmem_slot, kTmemCols);
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  tcgen05_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;

  if (warp == kWarpX) {
    // ------------------------------------------------------------ x producer
    if (lane == 0) {
      prefetch_tensormap(&map_x);
      const int nblk = F_in / 8;
      uint32_t b = 0;
      bool ok = true;
      for (int tile = pair; tile < args.ntiles && ok; tile += npairs) {
        const int row0 = tile * kTileTokens + (int)rank * kRowsPerCta;
        for (int q = 0; q < nblk; ++q, ++b) {
          const uint32_t s = b % kXStages, ph = (b / kXStages) & 1u;
          if (!mbar_wait_bounded(bar_x_empty(s), ph ^ 1u, fault, FAULT_WAIT_X_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_x_full(s), kXStageBytes);
          tma_load_2d(sX + s * kXStageBytes, &map_x, bar_x_full(s), q * 64, row0);
        }
      }
    }
  } else if (warp == kWarpB) {
    // ------------------------------------------------------------ B producer
    if (lane == 0) {
      prefetch_tensormap(&map_b16);
      prefetch_tensormap(&map_b32);
      prefetch_tensormap(&map_b64);
      const uint32_t leader_b_full0 = mapa_shared(bar_b_full(0), 0);
      uint32_t pc = 0;
      bool ok = true;
      for (int tile = pair; tile < args.ntiles && ok; tile += npairs) {
        for (int c = 0; c < nchunks && ok; ++c) {
          const int co = chunk_fields(F_out, c);
          for (int j = 0; j < kNumJobs && ok; ++j) {
            const JobDesc jd = job_desc(MODE, j);
            const int R = job_rows(jd, co);
            const int pieces = job_pieces(jd, F_in);
            const int64_t jbase = b_job_base(MODE, F_in, F_out, c, j);
            const CUtensorMap *map = R == 16 ? &map_b16 : (R == 32 ? &map_b32 : &map_b64);
            const uint32_t bytes = (uint32_t)R * 64u;
            for (int p = 0; p < pieces; ++p, ++pc) {
              const uint32_t s = pc % kBStages, ph = (pc / kBStages) & 1u;
              if (!mbar_wait_bounded(bar_b_empty(s), ph ^ 1u, fault, FAULT_WAIT_B_EMPTY,
                                     kWaitLimitNs)) {
                ok = false;
                break;
              }
              if (leader) mbar_arrive_expect_tx(bar_b_full(s), 2u * bytes);
              const int row = (int)(jbase + (int64_t)(p * 2 + (int)rank) * 4 * R);
              tma_load_2d_pair(sB + s * kBStageBytes, map, leader_b_full0 + 8u * s, 0, row);
            }
          }
        }
      }
      // the last panels' release (an MMA commit into this CTA) must land before exit
      if (ok) {
        const uint32_t first = pc > (uint32_t)kBStages ? pc - kBStages : 0u;
        for (uint32_t k = first; k < pc; ++k) {
          if (!mbar_wait_bounded(bar_b_empty(k % kBStages), (k / kBStages) & 1u, fault,
                                 FAULT_WAIT_B_EMPTY, kWaitLimitNs))
            break;
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issue
    if (leader && lane == 0) {
      uint32_t pc = 0, acc = 0, ti = 0;
      bool ok = true;
      for (int tile = pair; tile < args.ntiles && ok; tile += npairs, ++ti) {
        if (!mbar_wait_bounded(bar_a_full, ti & 1u, fault, FAULT_WAIT_A_FULL, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
        for (int c = 0; c < nchunks && ok; ++c, ++acc) {
          const int co = chunk_fields(F_out, c);
          const uint32_t buf = acc & 1u;
          if (!mbar_wait_bounded(bar_acc_empty(buf), ((acc >> 1) & 1u) ^ 1u, fault,
                                 FAULT_WAIT_ACC_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint32_t d_base = tmem_base + buf * kAccBufCols;
          for (int j = 0; j < kNumJobs && ok; ++j) {
            const JobDesc jd = job_desc(MODE, j);
            const int R = job_rows(jd, co);
            const int N = 2 * R;
            const uint32_t idesc = idesc_bf16_f32(128, N);
            const int pieces = job_pieces(jd, F_in);
            for (int p = 0; p < pieces; ++p, ++pc) {
              const uint32_t s = pc % kBStages, ph = (pc / kBStages) & 1u;
              if (!mbar_wait_bounded(bar_b_full(s), ph, fault, FAULT_WAIT_B_FULL, kWaitLimitNs)) {
                ok = false;
                break;
              }
              tcgen05_fence_after();
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                const uint64_t bdesc = smem_desc_kmajor_noswizzle(
                    sB + s * kBStageBytes + (uint32_t)(ks * 2 * R * 16), (uint32_t)R * 16u, 128u);
                for (int t = 0; t < jd.ntarget; ++t) {
                  const int kc = jd.acoord[t] * kcs + p * 4 + ks * 2;
                  const uint64_t adesc =
                      smem_desc_kmajor_noswizzle(sA + (uint32_t)kc * 1024u, 1024u, 128u);
                  mma_bf16_pair(d_base + (uint32_t)(jd.dgroup[t] * (co / 2)), adesc, bdesc, idesc,
                                (p > 0 || ks > 0) ? 1u : 0u);
                }
              }
              mma_commit_pair_mc(bar_b_empty(s), 0x3);
            }
          }
          if (ok) mma_commit_pair_mc(bar_acc_full(buf), 0x3);
        }
        if (ok) mma_commit_pair_mc(bar_a_empty, 0x3);
      }
    }
  } else if (warp >= kDftWarp0 && warp < kDftWarp0 + kNumDftWarps) {
    // ------------------------------------------------------------ forward transform
    const int grp = (warp - kDftWarp0) >> 1;
    const int t = ((warp - kDftWarp0) & 1) * 32 + lane;  // token row in this CTA
    const int nblk = F_in / 8;
    const uint32_t leader_a_full = mapa_shared(bar_a_full, 0);
    uint32_t ti = 0;
    bool ok = true;
    for (int tile = pair; tile < args.ntiles && ok; tile += npairs, ++ti) {
      if (ti > 0 &&
          !mbar_wait_bounded(bar_a_empty, (ti - 1) & 1u, fault, FAULT_WAIT_A_EMPTY, kWaitLimitNs)) {
        ok = false;
        break;
      }
      for (int q = grp; q < nblk; q += 2) {
        const uint32_t b = ti * (uint32_t)nblk + (uint32_t)q;
        const uint32_t s = b % kXStages, ph = (b / kXStages) & 1u;
        if (!mbar_wait_bounded(bar_x_full(s), ph, fault, FAULT_WAIT_X_FULL, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const uint8_t *xs = gbase + (sX - base) + s * kXStageBytes + t * 128;
        uint32_t out[8][4];
#pragma unroll
        for (int f = 0; f < 8; ++f) {
          const uint4 v = *reinterpret_cast<const uint4 *>(xs + ((f ^ (t & 7)) << 4));
          float xv[8], z[8];
          unpack_bf16x8(v, xv);
          if (MODE == kModeCyclic8)
            fwd_cyclic8(xv, z);
          else
            fwd_d8(xv, z);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (f & 1)
              out[c][f >> 1] |= pack_bf16x2(0.f, z[c]) & 0xFFFF0000u;
            else
              out[c][f >> 1] = pack_bf16x2(z[c], 0.f) & 0x0000FFFFu;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(bar_x_empty(s), rank));
        uint8_t *A = gbase + (size_t)t * 16;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(A + (size_t)(c * kcs + q) * 1024) =
              make_uint4(out[c][0], out[c][1], out[c][2], out[c][3]);
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_a_full);
    }
    // the release of the last tile's A (an MMA commit into this CTA) must land before exit
    if (ok && ti > 0)
      mbar_wait_bounded(bar_a_empty, (ti - 1) & 1u, fault, FAULT_WAIT_A_EMPTY, kWaitLimitNs);
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                // TMEM lane quarter of this warp
    const int row = (q4 & 1) * 32 + lane;   // token row in this CTA
    const int h = q4 >> 1;                  // which half of each chunk's fields
    const uint32_t leader_acc_empty0 = mapa_shared(bar_acc_empty(0), 0);
    uint32_t acc = 0;
    bool ok = true;
    for (int tile = pair; tile < args.ntiles && ok; tile += npairs) {
      const int64_t tok = (int64_t)tile * kTileTokens + (int64_t)rank * kRowsPerCta + row;
      const bool valid = tok < args.T;
      uint4 *yrow = reinterpret_cast<uint4 *>(args.y) + (valid ? tok * F_out : 0);
      for (int c = 0; c < nchunks; ++c, ++acc) {
        const int co = chunk_fields(F_out, c);
        const int half = co >> 1;
        const uint32_t buf = acc & 1u;
        if (!mbar_wait_bounded(bar_acc_full(buf), (acc >> 1) & 1u, fault, FAULT_WAIT_ACC_FULL,
                               kWaitLimitNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
        const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32) << 16) + buf * kAccBufCols;
        for (int fg = 0; fg < half; fg += 8) {
          uint32_t v[8][8];
#pragma unroll
          for (int k = 0; k < 8; ++k) tmem_ld_x8(tb + (uint32_t)(k * half + fg), v[k]);
          tmem_wait_ld();
#pragma unroll
          for (int f = 0; f < 8; ++f) {
            float z[8], yv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) z[group_coord(MODE, k)] = __uint_as_float(v[k][f]);
            if (MODE == kModeCyclic8)
              inv_cyclic8(z, yv);
            else
              inv_d8(z, yv);
            if (args.gelu) {
#pragma unroll
              for (int g = 0; g < 8; ++g) yv[g] = gelu_erf(yv[g]);
            }
            if (valid) {
              const int o = c * kCoMax + h * half + fg + f;
              yrow[o] = make_uint4(pack_bf16x2(yv[0], yv[1]), pack_bf16x2(yv[2], yv[3]),
                                   pack_bf16x2(yv[4], yv[5]), pack_bf16x2(yv[6], yv[7]));
            }
          }
        }
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + 8u * buf);
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  if (*(volatile unsigned int *)fault != 0u) {
    // a bounded wait gave up somewhere: give copies still in flight time to land
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kWarpMma) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- packing

struct D8Blocks {
  const __nv_bfloat16 *w[5];
};

// One CUDA block per (piece, CTA half) panel of job j of chunk c.
template <int MODE>
__global__ void pack_b_kernel(const __nv_bfloat16 *__restrict__ Wc, D8Blocks d8, int F_in,
                              int F_out, int c, int j, int64_t jbase,
                              __nv_bfloat16 *__restrict__ dst) {
  const JobDesc jd = job_desc(MODE, j);
  const int co = chunk_fields(F_out, c);
  const int R = job_rows(jd, co);
  const int p = blockIdx.x >> 1, hh = blockIdx.x & 1;
  const int64_t row0 = jbase + (int64_t)(p * 2 + hh) * 4 * R;
  const int nel = 4 * R * 8;
  for (int e = threadIdx.x; e < nel; e += blockDim.x) {
    const int kc = e / (R * 8);
    const int r = (e / 8) % R;
    const int el = e % 8;
    const int kk = p * kKPiece + kc * 8 + el;  // K index within the job
    // output coordinate / field of B row r in this CTA half
    int cout, o;
    if (jd.ncoord == 1) {
      cout = jd.acoord[0];
      o = c * kCoMax + hh * (co / 2) + r;
    } else {
      const int hc = co / 2;
      cout = jd.acoord[0] + (r >= hc ? 1 : 0);
      o = c * kCoMax + hh * hc + (r % hc);
    }
    const int cin = jd.acoord[0] + (kk >= F_in ? 1 : 0);
    const int i = kk % F_in;
    double val = 0.0;
    if (MODE == kModeCyclic8) {
      // bin of the coordinate pair and the real/imaginary parts of What_k[o, i]
      const int bin = cout == 0 ? 0 : (cout == 7 ? 4 : (cout + 1) / 2);
      double re = 0.0, im = 0.0;
      for (int m = 0; m < 8; ++m) {
        const double w = (double)__bfloat162float(Wc[((size_t)o * F_in + i) * 8 + m]);
        const double ang = 2.0 * M_PI * (double)((m * bin) % 8) / 8.0;
        re += w * cos(ang);
        im -= w * sin(ang);
      }
      re /= 8.0;
      im /= 8.0;
      if (bin == 0 || bin == 4) {
        val = re;
      } else {
        const bool out_re = (cout & 1) == 1, in_re = (cin & 1) == 1;
        // [Yr; Yi] = [[Wr, -Wi], [Wi, Wr]] [Xr; Xi], doubled for the one-sided inverse
        val = 2.0 * (out_re ? (in_re ? re : -im) : (in_re ? im : re));
      }
    } else {
      if (jd.ncoord == 1) {
        val = (double)__bfloat162float(d8.w[cout][(size_t)o * F_in + i]);
      } else {
        const int bo = (cout - jd.acoord[0]), bi = (cin - jd.acoord[0]);
        val = (double)__bfloat162float(d8.w[4][(size_t)(2 * o + bo) * (2 * F_in) + 2 * i + bi]);
      }
    }
    dst[(row0 + (int64_t)kc * R + r) * 8 + el] = __float2bfloat16_rn((float)val);
  }
}

template <int MODE>
int launch_pack(const __nv_bfloat16 *Wc, D8Blocks d8, int F_in, int F_out, void *dst,
                cudaStream_t s) {
  for (int c = 0; c < num_chunks(F_out); ++c) {
    for (int j = 0; j < kNumJobs; ++j) {
      const JobDesc jd = job_desc(MODE, j);
      const int64_t jb = b_job_base(MODE, F_in, F_out, c, j);
      const int blocks = job_pieces(jd, F_in) * 2;
      pack_b_kernel<MODE><<<blocks, 256, 0, s>>>(Wc, d8, F_in, F_out, c, j, jb,
                                                  static_cast<__nv_bfloat16 *>(dst));
    }
  }
  return check_launch("tensor-core weight packing");
}

// ---------------------------------------------------------------- host launch

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int make_map_2d(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer,
                uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle swz) {
  auto enc = get_encode_fn();
  if (!enc) return set_error(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return EQLIN_OK;
}

struct DevCache {
  int max_clusters[2] = {0, 0};
  bool attr_set[2] = {false, false};
};
std::mutex g_cache_mu;
DevCache g_cache[64];

template <int MODE>
int launch_tc(const void *x, const void *Bpack, void *y, int64_t T, int F_in, int F_out, int gelu,
              cudaStream_t s) {
  if (T >= (int64_t)0x7fffff00LL) return set_error(EQLIN_ERR_UNSUPPORTED, "T too large");
  const int ntiles = (int)((T + kTileTokens - 1) / kTileTokens);
  const size_t smem = smem_bytes_for(F_in);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(EQLIN_ERR_CUDA, "cudaGetDevice failed");
  auto kern = spectral8_tc_kernel<MODE>;
  int maxc = 0;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    DevCache &dc = g_cache[dev];
    if (!dc.attr_set[MODE]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)(1024 + kMaxFin * 1024 + kXStages * kXStageBytes +
                                                 kBStages * kBStageBytes + 256));
      if (e != cudaSuccess) return set_error(EQLIN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = 1024 + kMaxFin * 1024 + kXStages * kXStageBytes + kBStages * kBStageBytes + 256;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (e != cudaSuccess || n <= 0)
        return set_error(EQLIN_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s (n=%d)",
                         cudaGetErrorString(e), n);
      dc.max_clusters[MODE] = n;
      dc.attr_set[MODE] = true;
    }
    maxc = dc.max_clusters[MODE];
  }
  CUtensorMap mx, mb16, mb32, mb64;
  int rc = make_map_2d(&mx, x, (uint64_t)F_in * 8, (uint64_t)T, (uint64_t)F_in * 16, 64,
                       kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  const int64_t rows = b_job_base(MODE, F_in, F_out, num_chunks(F_out), 0);
  rc = make_map_2d(&mb16, Bpack, 8, (uint64_t)rows, 16, 8, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = make_map_2d(&mb32, Bpack, 8, (uint64_t)rows, 16, 8, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = make_map_2d(&mb64, Bpack, 8, (uint64_t)rows, 16, 8, 256, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;

  TcArgs a;
  a.T = T;
  a.F_in = F_in;
  a.F_out = F_out;
  a.ntiles = ntiles;
  a.gelu = gelu;
  a.y = static_cast<__nv_bfloat16 *>(y);
  const int npairs = ntiles < maxc ? ntiles : maxc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * npairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mx, mb16, mb32, mb64, a);
  if (e != cudaSuccess) return set_error(EQLIN_ERR_CUDA, "tensor-core launch: %s", cudaGetErrorString(e));
  return check_launch("spectral8_tc_kernel");
}

}  // namespace

// ---------------------------------------------------------------- interface

bool cyclic_tc_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && N == 8 && Cin % kKPiece == 0 && Cin >= kKPiece && Cin <= kMaxFin &&
         Cout % 32 == 0 && Cout >= 32;
}

bool d8_tc_supported(int C, int dtype) {
  const int F = C / 8;
  return dtype == EQLIN_BF16 && C % 8 == 0 && F % kKPiece == 0 && F >= kKPiece && F <= kMaxFin;
}

size_t cyclic_tc_bytes(int, int Cin, int Cout) {
  return (size_t)b_job_base(kModeCyclic8, Cin, Cout, num_chunks(Cout), 0) * 16;
}

size_t d8_tc_bytes(int C) {
  const int F = C / 8;
  return (size_t)b_job_base(kModeD8, F, F, num_chunks(F), 0) * 16;
}

int launch_cyclic_tc_pack(const void *W, int, int Cin, int Cout, void *dst, cudaStream_t s) {
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  return launch_pack<kModeCyclic8>(static_cast<const __nv_bfloat16 *>(W), none, Cin, Cout, dst, s);
}

int launch_d8_tc_pack(const void *const w[5], int C, void *dst, cudaStream_t s) {
  D8Blocks d8;
  for (int k = 0; k < 5; ++k) d8.w[k] = static_cast<const __nv_bfloat16 *>(w[k]);
  return launch_pack<kModeD8>(nullptr, d8, C / 8, C / 8, dst, s);
}

int launch_cyclic_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                     cudaStream_t s) {
  return launch_tc<kModeCyclic8>(x, Bpack, y, T, Cin, Cout, 0, s);
}

int launch_d8_tc(const void *x, const void *Bpack, void *y, int64_t T, int C, int gelu,
                 cudaStream_t s) {
  return launch_tc<kModeD8>(x, Bpack, y, T, C / 8, C / 8, gelu, s);
}

}  // namespace eqlin
