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

// warp roles.  Two MMA issuers (one per TMEM accumulator buffer; a single
// issuing thread cannot keep the tensor pipe busy with M=128 pair
// instructions), each fed by its own weight-panel producer and ring.
constexpr int kThreads = 512;
constexpr int kWarpB0 = 0;     // weight-panel producer for ring / buffer 0
constexpr int kWarpMma0 = 1;   // MMA issuer for buffer 0; TMEM allocation
constexpr int kWarpB1 = 2;     // weight-panel producer for ring / buffer 1
constexpr int kWarpMma1 = 3;   // MMA issuer for buffer 1
constexpr int kDftWarp0 = 4;   // x TMA loads + in-place forward transform
constexpr int kNumDftWarps = 8;
constexpr int kEpiWarp0 = 12;  // TMEM -> inverse transform -> y
constexpr int kNumEpiWarps = 4;

constexpr int kRowsPerCta = 64;
constexpr int kTileTokens = 2 * kRowsPerCta;
constexpr int kBlockBytes = kRowsPerCta * 128;  // one 8-field block of A: 64 rows x 128 B
constexpr int kBStages = 6;       // 2 rings of kRingStages
constexpr int kRingStages = 3;
constexpr int kBStageBytes = 8192;
constexpr int kStageBufBytes = 2048;  // epilogue staging: 32 token rows x 4 fields x 16 B
constexpr int kStagingBytes = kNumEpiWarps * 2 * kStageBufBytes;
constexpr int kCoMax = 64;     // output fields per chunk
constexpr int kMaxFin = 160;   // A operand = Fin KB of shared memory
constexpr int kMaxBlocks = kMaxFin / 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccBufCols = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kSleepNs = 128;   // back-off of warps that wait for long phases
constexpr int kNumJobs = 5;
constexpr int kNumBMaps = 16;  // panel TMA boxes of 0.5..8 KB (4..64 rows of 128 B)

// A "job" is one block product over all input fields.  Its K-steps (16 bf16
// each) read two adjacent 16-byte chunks of one 128-byte row of the A operand:
//   real   : one coordinate over 16 fields, K-step i = blocks (2i, 2i+1),
//            chunk pair `pair` of row 2i + blk_off;  B rows = chunk/2 fields
//   paired : two coordinates over 8 fields, K-step i = block i, chunk pair
//            `pair`; B rows = 2 coordinates x chunk/2 fields
struct JobDesc {
  int paired;     // 0 real, 1 paired
  int ntarget;    // A/D targets sharing one B panel
  int blk_off[2]; // real jobs: which block of the pair holds the chunk pair
  int pair[2];    // chunk pair index (0..3) within the 128-byte row
  int dgroup[2];  // first TMEM column group (units of chunk/2 columns)
  int bstyle;     // 0: B = [kc][R rows][8]; 1: B = [Wi | Wr | -Wi] rows (cyclic bins)
};

__host__ __device__ inline JobDesc job_desc(int mode, int j) {
  if (mode == kModeCyclic8) {
    switch (j) {
      case 0: return {0, 1, {0, 0}, {0, 0}, {0, 0}, 0};  // Re X0
      case 1: return {0, 1, {1, 0}, {0, 0}, {1, 0}, 0};  // Re X4
      case 2: return {1, 1, {0, 0}, {1, 0}, {2, 0}, 1};  // X1
      case 3: return {1, 1, {0, 0}, {2, 0}, {4, 0}, 1};  // X2
      default: return {1, 1, {0, 0}, {3, 0}, {6, 0}, 1}; // X3
    }
  }
  switch (j) {
    case 0: return {0, 1, {0, 0}, {0, 0}, {0, 0}, 0};  // A1
    case 1: return {0, 1, {0, 0}, {1, 0}, {1, 0}, 0};  // A2
    case 2: return {0, 1, {1, 0}, {0, 0}, {2, 0}, 0};  // B1
    case 3: return {0, 1, {1, 0}, {1, 0}, {3, 0}, 0};  // B2
    default: return {1, 2, {0, 0}, {2, 3}, {4, 6}, 0}; // E, rows a = 0 and a = 1
  }
}

// Issuer of job j: each chunk's jobs are split so both issuers issue 40
// K-steps per full chunk (cyclic: Re X0, Re X4, X1 | X2, X3; D8: A1, A2, B1,
// B2 | E on both rows).
__host__ __device__ inline int job_issuer(int mode, int j) {
  return mode == kModeCyclic8 ? (j < 3 ? 0 : 1) : (j < 4 ? 0 : 1);
}

// Coordinate held by TMEM column group k (k = 0..7) of an accumulator buffer:
// cyclic [Re Y0, Re Y4, Im Y1, Re Y1, Im Y2, Re Y2, Im Y3, Re Y3] (the complex
// bins' B rows are ordered [Im; Re]); D8 in coordinate order.
__host__ __device__ inline int group_coord(int mode, int k) {
  if (mode == kModeCyclic8) {
    const int map[8] = {0, 7, 2, 1, 4, 3, 6, 5};
    return map[k];
  }
  return k;
}

__host__ __device__ inline int chunk_fields(int F_out, int c) {
  const int r = F_out - c * kCoMax;
  return r < kCoMax ? r : kCoMax;
}
__host__ __device__ inline int num_chunks(int F_out) { return (F_out + kCoMax - 1) / kCoMax; }
__host__ __device__ inline int job_rows(const JobDesc &jd, int co) { return jd.paired ? co : co / 2; }
__host__ __device__ inline int job_ksteps(const JobDesc &jd, int F_in) {
  return jd.paired ? F_in / 8 : F_in / 16;
}
__host__ __device__ inline int kstep_bytes(const JobDesc &jd, int R) {
  return jd.bstyle ? 24 * R : 32 * R;
}
// K-steps per B stage: the largest divisor of the job's K-step count whose
// panel is a multiple of 512 bytes and fits one stage (0 if none exists).
__host__ __device__ inline int stage_ksteps(const JobDesc &jd, int F_in, int co) {
  const int n = job_ksteps(jd, F_in);
  const int kb = kstep_bytes(jd, job_rows(jd, co));
  for (int g = n; g >= 1; --g)
    if (n % g == 0 && g * kb <= kBStageBytes && (g * kb) % 512 == 0) return g;
  return 0;
}

// Byte offset of the packed panels of (chunk c, job j).  A job's panels are
// ordered (stage, CTA half), each the shared-memory image of one B stage.
// Called with (c = nchunks, j = 0) it returns the total size.
__host__ __device__ inline int64_t b_job_offset(int mode, int F_in, int F_out, int c, int j) {
  int64_t off = 0;
  const int nch = num_chunks(F_out);
  for (int cc = 0; cc < nch; ++cc) {
    const int co = chunk_fields(F_out, cc);
    for (int jj = 0; jj < kNumJobs; ++jj) {
      if (cc == c && jj == j) return off;
      const JobDesc jd = job_desc(mode, jj);
      off += (int64_t)2 * job_ksteps(jd, F_in) * kstep_bytes(jd, job_rows(jd, co));
    }
  }
  return off;
}

bool tc_shape_ok(int mode, int F_in, int F_out) {
  if (F_in < 16 || F_in > kMaxFin || F_in % 16 || F_out < 32 || F_out % 32) return false;
  for (int c = 0; c < num_chunks(F_out); ++c)
    for (int j = 0; j < kNumJobs; ++j)
      if (stage_ksteps(job_desc(mode, j), F_in, chunk_fields(F_out, c)) == 0) return false;
  return true;
}

constexpr int kCtrlBytes = 1024;  // barriers, TMEM address, job plan

size_t smem_bytes_for(int F_in) {
  return 1024 + (size_t)F_in * 1024 + kBStages * kBStageBytes + kStagingBytes + kCtrlBytes;
}

// Per-job schedule, identical for every full chunk (64 fields) and computed
// separately for a shorter last chunk; built once per CTA in the prologue.
struct JobPlan {
  uint32_t off;    // byte offset of the job's panels within its chunk
  uint32_t bytes;  // bytes of one stage (one CTA half)
  uint16_t G;      // K-steps per stage
  uint16_t nst;    // stages
  uint16_t kb;     // bytes per K-step
  uint16_t R;      // B rows per CTA half
};
static_assert(sizeof(JobPlan) == 16, "JobPlan layout");
constexpr int kPlanOffset = 512;  // within the control block

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

// Weight-panel TMA maps: the packed buffer viewed as rows of 128 bytes, box
// heights 4, 8, ..., 64 rows (0.5 to 8 KB).
struct BMaps {
  CUtensorMap m[kNumBMaps];
};

// In-place forward transform of one token's two 128-byte rows (blocks q0 =
// 2j and q1 = 2j+1, 16 fields).  On entry chunk f of a row holds field f's 8
// slots; on exit the rows hold the chunk pairs the MMA K-steps read:
//   cyclic  row q0: [X0(q0) X0(q1)] [ReX1 ImX1](q0) [ReX2 ImX2](q0) [ReX3 ImX3](q0)
//           row q1: [X4(q0) X4(q1)] [ReX1 ImX1](q1) [ReX2 ImX2](q1) [ReX3 ImX3](q1)
//   D8      row q0: [A1(q0) A1(q1)] [A2(q0) A2(q1)] [E00 E01](q0) [E10 E11](q0)
//           row q1: [B1(q0) B1(q1)] [B2(q0) B2(q1)] [E00 E01](q1) [E10 E11](q1)
// where "X(q)" is one coordinate of the 8 fields of block q as 8 bf16.
template <int MODE>
__device__ __forceinline__ void transform_block(const uint4 (&in)[8], uint32_t (&out)[8][4]) {
#pragma unroll
  for (int f = 0; f < 8; f += 2) {
    float xa[8], xb[8], za[8], zb[8];
    unpack_bf16x8(in[f], xa);
    unpack_bf16x8(in[f + 1], xb);
    if (MODE == kModeCyclic8) {
      fwd_cyclic8(xa, za);
      fwd_cyclic8(xb, zb);
    } else {
      fwd_d8(xa, za);
      fwd_d8(xb, zb);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) out[c][f >> 1] = pack_bf16x2(za[c], zb[c]);
  }
}

template <int MODE>
__device__ __forceinline__ void transform_rows(uint8_t *row0, uint8_t *row1, int sw) {
  auto put = [&](uint8_t *row, int slot, const uint32_t (&v)[4]) {
    *reinterpret_cast<uint4 *>(row + ((slot ^ sw) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
  };
  uint4 in0[8], in1[8];
#pragma unroll
  for (int f = 0; f < 8; ++f) {
    in0[f] = *reinterpret_cast<const uint4 *>(row0 + ((f ^ sw) << 4));
    in1[f] = *reinterpret_cast<const uint4 *>(row1 + ((f ^ sw) << 4));
  }
  // every input chunk is in registers now, so outputs may overwrite them
  uint32_t out[8][4];
  transform_block<MODE>(in0, out);          // block q0
  if (MODE == kModeCyclic8) {
    put(row0, 0, out[0]);
    put(row1, 0, out[7]);
#pragma unroll
    for (int c = 1; c <= 6; ++c) put(row0, c + 1, out[c]);
  } else {
    put(row0, 0, out[0]);
    put(row0, 2, out[1]);
    put(row1, 0, out[2]);
    put(row1, 2, out[3]);
#pragma unroll
    for (int c = 4; c < 8; ++c) put(row0, c, out[c]);
  }
  transform_block<MODE>(in1, out);          // block q1
  if (MODE == kModeCyclic8) {
    put(row0, 1, out[0]);
    put(row1, 1, out[7]);
#pragma unroll
    for (int c = 1; c <= 6; ++c) put(row1, c + 1, out[c]);
  } else {
    put(row0, 1, out[0]);
    put(row0, 3, out[1]);
    put(row1, 1, out[2]);
    put(row1, 3, out[3]);
#pragma unroll
    for (int c = 4; c < 8; ++c) put(row1, c, out[c]);
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    spectral8_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_y,
                        const __grid_constant__ BMaps bmaps, const TcArgs args) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);

  const int F_in = args.F_in;
  const int F_out = args.F_out;
  const int nchunks = num_chunks(F_out);
  const int nblk = F_in / 8;  // 8-field blocks of A

  const uint32_t sA = base;
  const uint32_t sB = sA + (uint32_t)F_in * 1024u;
  const uint32_t sStage = sB + kBStages * kBStageBytes;
  const uint32_t sBar = sStage + kStagingBytes;
  auto bar_x_full = [&](int q) { return sBar + 8u * q; };                     // kMaxBlocks
  auto bar_b_full = [&](int i) { return sBar + 8u * (kMaxBlocks + i); };      // kBStages
  auto bar_b_empty = [&](int i) { return sBar + 8u * (kMaxBlocks + kBStages + i); };
  auto bar_acc_full = [&](int i) { return sBar + 8u * (kMaxBlocks + 2 * kBStages + i); };
  auto bar_acc_empty = [&](int i) { return sBar + 8u * (kMaxBlocks + 2 * kBStages + 2 + i); };
  const uint32_t bar_a_full = sBar + 8u * (kMaxBlocks + 2 * kBStages + 4);
  const uint32_t bar_a_empty = sBar + 8u * (kMaxBlocks + 2 * kBStages + 5);
  const uint32_t tmem_slot = sBar + 8u * (kMaxBlocks + 2 * kBStages + 6);
  volatile uint32_t *tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t *>(gbase + (tmem_slot - base));
  // plan[0][j]: jobs of a full chunk, plan[1][j]: jobs of the last chunk
  JobPlan (*plan)[kNumJobs] = reinterpret_cast<JobPlan (*)[kNumJobs]>(gbase + (sBar - base) + kPlanOffset);
  uint32_t *chunk_bytes_ptr = reinterpret_cast<uint32_t *>(gbase + (sBar - base) + kPlanOffset - 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  unsigned int *fault = &g_fault_word;

  if (threadIdx.x == 0) {
    for (int q = 0; q < kMaxBlocks; ++q) mbar_init(bar_x_full(q), 1);
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(bar_b_full(i), 1);
      mbar_init(bar_b_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc_full(i), 2);                 // one commit per issuer
      mbar_init(bar_acc_empty(i), 2 * kNumEpiWarps);
    }
    mbar_init(bar_a_full, 2 * kNumDftWarps);
    mbar_init(bar_a_empty, 2);                       // one commit per issuer
    fence_mbarrier_init_cluster();
    for (int tp = 0; tp < 2; ++tp) {
      const int co = tp == 0 ? (F_out < kCoMax ? F_out : kCoMax) : chunk_fields(F_out, nchunks - 1);
      uint32_t off = 0;
      for (int j = 0; j < kNumJobs; ++j) {
        const JobDesc jd = job_desc(MODE, j);
        const int R = job_rows(jd, co);
        const int kb = kstep_bytes(jd, R);
        const int G = stage_ksteps(jd, F_in, co);
        const int nst = G > 0 ? job_ksteps(jd, F_in) / G : 0;
        plan[tp][j] = {off, (uint32_t)(G * kb), (uint16_t)G, (uint16_t)nst, (uint16_t)kb, (uint16_t)R};
        off += 2u * (uint32_t)(nst * G * kb);
      }
      if (tp == 0) *chunk_bytes_ptr = off;
    }
  }
  if (warp == kWarpMma0) tmem_alloc_pair(tmem_slot, kTmemCols);
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  tcgen05_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  const int ntile_local = args.ntiles > pair ? (args.ntiles - pair + npairs - 1) / npairs : 0;
  const int total_chunks = ntile_local * nchunks;  // global chunk index g = tile_iter * nchunks + c

  if (warp == kWarpB0 || warp == kWarpB1) {
    // ------------------------------------------------------------ weight-panel producers
    // Producer r streams the panels of issuer r's jobs of every chunk into ring r.
    if (lane == 0) {
      const int r = warp == kWarpB0 ? 0 : 1;
      for (int k = 0; k < kNumBMaps; ++k) prefetch_tensormap(&bmaps.m[k]);
      const uint32_t leader_b_full0 = mapa_shared(bar_b_full(0), 0);
      const uint32_t chunk_bytes = *chunk_bytes_ptr;
      uint32_t pc = 0;
      bool ok = true;
      for (int g = 0; g < total_chunks && ok; ++g) {
        const int c = g % nchunks;
        const JobPlan *pl = plan[c == nchunks - 1 ? 1 : 0];
        for (int j = 0; j < kNumJobs && ok; ++j) {
          if (job_issuer(MODE, j) != r) continue;
          const JobPlan p = pl[j];
          const CUtensorMap *map = &bmaps.m[p.bytes / 512 - 1];
          uint32_t off = (uint32_t)c * chunk_bytes + p.off + rank * p.bytes;
          for (int st = 0; st < p.nst; ++st, ++pc, off += 2u * p.bytes) {
            const uint32_t slot = (uint32_t)r * kRingStages + pc % kRingStages;
            const uint32_t ph = (pc / kRingStages) & 1u;
            if (!mbar_wait_bounded(bar_b_empty(slot), ph ^ 1u, fault, FAULT_WAIT_B_EMPTY,
                                   kWaitLimitNs, kSleepNs / 4)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(bar_b_full(slot), 2u * p.bytes);
            tma_load_2d_pair(sB + slot * kBStageBytes, map, leader_b_full0 + 8u * slot, 0,
                             (int32_t)(off / 128u));
          }
        }
      }
      // the last panels' release (an MMA commit into this CTA) must land before exit
      if (ok) {
        const uint32_t first = pc > (uint32_t)kRingStages ? pc - kRingStages : 0u;
        for (uint32_t k = first; k < pc; ++k)
          if (!mbar_wait_bounded(bar_b_empty((uint32_t)r * kRingStages + k % kRingStages),
                                 (k / kRingStages) & 1u, fault, FAULT_WAIT_B_EMPTY, kWaitLimitNs))
            break;
      }
    }
  } else if (warp == kWarpMma0 || warp == kWarpMma1) {
    // ------------------------------------------------------------ MMA issue (leader CTA)
    if (leader && lane == 0) {
      const int r = warp == kWarpMma0 ? 0 : 1;
      const uint64_t a_desc_base = smem_desc_kmajor_sw128(sA);
      // descriptor of this ring's first stage without the leading byte offset
      // (set per job); stage k adds k * kBStageBytes / 16 to the start address
      const uint64_t ring_desc = smem_desc_kmajor_noswizzle(sB + (uint32_t)r * kRingStages * kBStageBytes, 0u, 128u);
      uint32_t pc = 0;
      int last_tile = -1;
      bool ok = true;
      for (int g = 0; g < total_chunks && ok; ++g) {
        const int ti = g / nchunks;
        const int c = g % nchunks;
        if (ti != last_tile) {
          if (!mbar_wait_bounded(bar_a_full, (uint32_t)ti & 1u, fault, FAULT_WAIT_A_FULL,
                                 kWaitLimitNs)) {
            ok = false;
            break;
          }
          last_tile = ti;
        }
        const int co = chunk_fields(F_out, c);
        const uint32_t buf = (uint32_t)g & 1u;
        if (!mbar_wait_bounded(bar_acc_empty(buf), (((uint32_t)g >> 1) & 1u) ^ 1u, fault,
                               FAULT_WAIT_ACC_EMPTY, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d_base = tmem_base + buf * kAccBufCols;
        const JobPlan *pl = plan[c == nchunks - 1 ? 1 : 0];
        for (int j = 0; j < kNumJobs && ok; ++j) {
          if (job_issuer(MODE, j) != r) continue;
          const JobDesc jd = job_desc(MODE, j);
          const JobPlan p = pl[j];
          const uint32_t R = p.R;
          const uint32_t idesc = idesc_bf16_f32(128, 2 * (int)R);
          const uint64_t lbo_field = (uint64_t)(((jd.bstyle ? (R / 2) * 16u : R * 16u) >> 4) & 0x3FFFu) << 16;
          const uint32_t d0 = d_base + (uint32_t)(jd.dgroup[0] * (co / 2));
          const uint32_t d1 = d_base + (uint32_t)(jd.dgroup[1] * (co / 2));
          const uint64_t a_step = jd.paired ? (kBlockBytes >> 4) : 2 * (kBlockBytes >> 4);
          uint64_t a0 = a_desc_base + (uint64_t)(jd.blk_off[0] * (kBlockBytes >> 4) + jd.pair[0] * 2);
          uint64_t a1 = a_desc_base + (uint64_t)(jd.blk_off[1] * (kBlockBytes >> 4) + jd.pair[1] * 2);
          const uint64_t b_step = (uint64_t)(p.kb >> 4);
          const int G = p.G;
          uint32_t accum = 0u;
          for (int st = 0; st < p.nst; ++st, ++pc) {
            const uint32_t k = pc % kRingStages;
            const uint32_t slot = (uint32_t)r * kRingStages + k;
            if (!mbar_wait_bounded(bar_b_full(slot), (pc / kRingStages) & 1u, fault,
                                   FAULT_WAIT_B_FULL, kWaitLimitNs)) {
              ok = false;
              break;
            }
            uint64_t bdesc = (ring_desc + (uint64_t)(k * (kBStageBytes >> 4))) | lbo_field;
            if (jd.ntarget == 1) {
#pragma unroll 4
              for (int i = 0; i < G; ++i) {
                mma_bf16_pair(d0, a0, bdesc, idesc, accum);
                a0 += a_step;
                bdesc += b_step;
                accum = 1u;
              }
            } else {
#pragma unroll 4
              for (int i = 0; i < G; ++i) {
                mma_bf16_pair(d0, a0, bdesc, idesc, accum);
                mma_bf16_pair(d1, a1, bdesc, idesc, accum);
                a0 += a_step;
                a1 += a_step;
                bdesc += b_step;
                accum = 1u;
              }
            }
            mma_commit_pair_mc(bar_b_empty(slot), 0x3);
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(bar_acc_full(buf), 0x3);
        // the tile's last chunk: this issuer's MMAs no longer need A
        if (c == nchunks - 1) mma_commit_pair_mc(bar_a_empty, 0x3);
      }
    }
  } else if (warp >= kDftWarp0 && warp < kDftWarp0 + kNumDftWarps) {
    // ------------------------------------------------------------ x loads + forward transform
    // Group grp (2 warps, 64 token rows) owns block pairs jp = grp, grp+4, ...:
    // its first lane loads them by TMA once the previous tile's MMAs have
    // released A, then all 64 threads transform them in place.
    constexpr int kGroups = kNumDftWarps / 2;
    const int grp = (warp - kDftWarp0) >> 1;
    const bool loader = ((warp - kDftWarp0) & 1) == 0 && lane == 0;
    const int t = ((warp - kDftWarp0) & 1) * 32 + lane;  // token row in this CTA
    const uint32_t leader_a_full = mapa_shared(bar_a_full, 0);
    if (loader) prefetch_tensormap(&map_x);
    uint32_t ti = 0;
    bool ok = true;
    for (int tile = pair; tile < args.ntiles && ok; tile += npairs, ++ti) {
      if (loader) {
        if (ti > 0 &&
            !mbar_wait_bounded(bar_a_empty, (ti - 1) & 1u, fault, FAULT_WAIT_A_EMPTY, kWaitLimitNs,
                               kSleepNs))
          ok = false;
        const int row0 = tile * kTileTokens + (int)rank * kRowsPerCta;
        for (int jp = grp; ok && jp < nblk / 2; jp += kGroups) {
          for (int h = 0; h < 2; ++h) {
            const int q = 2 * jp + h;
            mbar_arrive_expect_tx(bar_x_full(q), kBlockBytes);
            tma_load_2d(sA + (uint32_t)q * kBlockBytes, &map_x, bar_x_full(q), q * 64, row0);
          }
        }
      }
      __syncwarp();
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int jp = grp; ok && jp < nblk / 2; jp += kGroups) {
        if (!mbar_wait_bounded(bar_x_full(2 * jp), ti & 1u, fault, FAULT_WAIT_X_FULL, kWaitLimitNs,
                               kSleepNs) ||
            !mbar_wait_bounded(bar_x_full(2 * jp + 1), ti & 1u, fault, FAULT_WAIT_X_FULL,
                               kWaitLimitNs, kSleepNs)) {
          ok = false;
          break;
        }
        uint8_t *r0 = gbase + (size_t)(2 * jp) * kBlockBytes + t * 128;
        transform_rows<MODE>(r0, r0 + kBlockBytes, t & 7);
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_a_full);
    }
    // the release of the last tile's A (an MMA commit into this CTA) must land before exit
    if (loader && ok && ti > 0)
      mbar_wait_bounded(bar_a_empty, (ti - 1) & 1u, fault, FAULT_WAIT_A_EMPTY, kWaitLimitNs);
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // Warp e reads TMEM lanes 32*(e%4).., i.e. token rows 32*(e%2).. of this
    // CTA and the first (e < 2) or second half of each chunk's fields; results
    // go through a 128-byte-swizzle-free 64-byte-swizzled staging buffer to
    // 2-D TMA stores of 32 tokens x 4 fields.
    const int e = warp - kEpiWarp0;
    const int q4 = warp & 3;                // TMEM lane quarter of this warp
    const int h = q4 >> 1;                  // which half of each chunk's fields
    const uint32_t leader_acc_empty0 = mapa_shared(bar_acc_empty(0), 0);
    const uint32_t stage0 = sStage + (uint32_t)(e * 2) * kStageBufBytes;
    uint8_t *const stage_ptr0 = gbase + (stage0 - base);
    const int sw = (lane >> 1) & 3;         // 64-byte swizzle of this lane's staging row
    if (lane == 0) prefetch_tensormap(&map_y);
    uint32_t nstore = 0;
    bool ok = true;
    for (int g = 0; g < total_chunks && ok; ++g) {
      const int tile = pair + (g / nchunks) * npairs;
      const int c = g % nchunks;
      const int row_base = tile * kTileTokens + (int)rank * kRowsPerCta + (q4 & 1) * 32;
      const int co = chunk_fields(F_out, c);
      const int half = co >> 1;
      const uint32_t buf = (uint32_t)g & 1u;
      if (!mbar_wait_bounded(bar_acc_full(buf), ((uint32_t)g >> 1) & 1u, fault,
                             FAULT_WAIT_ACC_FULL, kWaitLimitNs, kSleepNs)) {
        ok = false;
        break;
      }
      tcgen05_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32) << 16) + buf * kAccBufCols;
      uint32_t vn[8][4];
#pragma unroll
      for (int k = 0; k < 8; ++k) tmem_ld_x4(tb + (uint32_t)(k * half), vn[k]);
      for (int fg = 0; fg < half; fg += 4, ++nstore) {
        tmem_wait_ld();
        uint32_t v[8][4];
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
          for (int f = 0; f < 4; ++f) v[k][f] = vn[k][f];
        if (fg + 4 < half) {
#pragma unroll
          for (int k = 0; k < 8; ++k) tmem_ld_x4(tb + (uint32_t)(k * half + fg + 4), vn[k]);
        }
        uint4 outv[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          float z[8], yv[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) z[group_coord(MODE, k)] = __uint_as_float(v[k][f]);
          if (MODE == kModeCyclic8)
            inv_cyclic8(z, yv);
          else
            inv_d8(z, yv);
          if (args.gelu) {
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) yv[gg] = gelu_erf(yv[gg]);
          }
          outv[f] = make_uint4(pack_bf16x2(yv[0], yv[1]), pack_bf16x2(yv[2], yv[3]),
                               pack_bf16x2(yv[4], yv[5]), pack_bf16x2(yv[6], yv[7]));
        }
        // staging buffer of this batch: free once the store two batches ago has read it
        const uint32_t sb = nstore & 1u;
        if (nstore >= 2) {
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
        }
        uint8_t *st = stage_ptr0 + sb * kStageBufBytes + lane * 64;
#pragma unroll
        for (int f = 0; f < 4; ++f) *reinterpret_cast<uint4 *>(st + ((f ^ sw) << 4)) = outv[f];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&map_y, stage0 + sb * kStageBufBytes, (c * kCoMax + h * half + fg) * 8, row_base);
          bulk_commit_group();
        }
      }
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + 8u * buf);
    }
    // stores must be complete before the CTA exits
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
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
  if (warp == kWarpMma0) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- packing

struct D8Blocks {
  const __nv_bfloat16 *w[5];
};

// Value of the spectral block matrix: output coordinate cout of field o from
// input coordinate cin of field i (cyclic coordinates as in fwd_cyclic8, with
// the complex bins doubled for the one-sided inverse; D8 coordinates A1, A2,
// B1, B2, E00, E01, E10, E11).
template <int MODE>
__device__ double block_value(const __nv_bfloat16 *Wc, const D8Blocks &d8, int F_in, int cout,
                              int o, int cin, int i) {
  if (MODE == kModeCyclic8) {
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
    if (bin == 0 || bin == 4) return re;
    const bool out_re = (cout & 1) == 1, in_re = (cin & 1) == 1;
    // [Yr; Yi] = [[Wr, -Wi], [Wi, Wr]] [Xr; Xi]
    return 2.0 * (out_re ? (in_re ? re : -im) : (in_re ? im : re));
  }
  if (cout < 4) return (double)__bfloat162float(d8.w[cout][(size_t)o * F_in + i]);
  const int bo = (cout - 4) & 1, bi = (cin - 4) & 1;
  return (double)__bfloat162float(d8.w[4][(size_t)(2 * o + bo) * (2 * F_in) + 2 * i + bi]);
}

// One CUDA block per (stage, CTA half) panel of job j of chunk c; thread loop
// over the panel's bf16 elements in shared-memory image order.
template <int MODE>
__global__ void pack_b_kernel(const __nv_bfloat16 *__restrict__ Wc, D8Blocks d8, int F_in,
                              int F_out, int c, int j, int64_t joff,
                              __nv_bfloat16 *__restrict__ dst) {
  const JobDesc jd = job_desc(MODE, j);
  const int co = chunk_fields(F_out, c);
  const int R = job_rows(jd, co);
  const int G = stage_ksteps(jd, F_in, co);
  const int kb = kstep_bytes(jd, R);
  const int st = blockIdx.x >> 1, hh = blockIdx.x & 1;
  const int64_t off = joff + (int64_t)(st * 2 + hh) * G * kb;   // bytes
  const int nel = G * kb / 2;
  const int hc = co / 2;
  // cyclic and D8 real-job coordinates in A order
  int coord_real;
  if (MODE == kModeCyclic8) coord_real = jd.blk_off[0] ? 7 : 0;
  else coord_real = (jd.blk_off[0] ? 2 : 0) + jd.pair[0];
  for (int e = threadIdx.x; e < nel; e += blockDim.x) {
    const int ks = st * G + (e * 2) / kb;        // K-step of the job
    const int w = e - ((e * 2) / kb) * (kb / 2); // element within the K-step panel
    double val;
    if (!jd.paired) {
      // [kc][R][8]: kc selects block 2ks + kc, row r -> output field
      const int kc = w / (R * 8), r = (w / 8) % R, el = w % 8;
      const int o = c * kCoMax + hh * hc + r;
      const int i = (2 * ks + kc) * 8 + el;
      val = block_value<MODE>(Wc, d8, F_in, coord_real, o, coord_real, i);
    } else if (jd.bstyle == 1) {
      // cyclic bin k: rows [Wi | Wr | -Wi] x 8 input fields of block ks
      const int blk = w / (hc * 8), r = (w / 8) % hc, el = w % 8;
      const int o = c * kCoMax + hh * hc + r;
      const int i = ks * 8 + el;
      const int cre = 2 * jd.pair[0] - 1, cim = 2 * jd.pair[0];   // Re, Im coordinates of the bin
      // Wi = value(Im <- Re), Wr = value(Re <- Re), -Wi = value(Re <- Im)
      val = blk == 0 ? block_value<MODE>(Wc, d8, F_in, cim, o, cre, i)
                     : (blk == 1 ? block_value<MODE>(Wc, d8, F_in, cre, o, cre, i)
                                 : block_value<MODE>(Wc, d8, F_in, cre, o, cim, i));
    } else {
      // D8 E: [kc = b][R rows = (b', field)][8 fields of block ks]
      const int kc = w / (R * 8), r = (w / 8) % R, el = w % 8;
      const int bo = r >= hc ? 1 : 0;
      const int o = c * kCoMax + hh * hc + (r % hc);
      const int i = ks * 8 + el;
      val = block_value<MODE>(Wc, d8, F_in, 4 + bo, o, 4 + kc, i);
    }
    dst[off / 2 + e] = __float2bfloat16_rn((float)val);
  }
}

template <int MODE>
int launch_pack(const __nv_bfloat16 *Wc, D8Blocks d8, int F_in, int F_out, void *dst,
                cudaStream_t s) {
  for (int c = 0; c < num_chunks(F_out); ++c) {
    for (int j = 0; j < kNumJobs; ++j) {
      const JobDesc jd = job_desc(MODE, j);
      const int co = chunk_fields(F_out, c);
      const int G = stage_ksteps(jd, F_in, co);
      const int64_t joff = b_job_offset(MODE, F_in, F_out, c, j);
      const int blocks = job_ksteps(jd, F_in) / G * 2;
      pack_b_kernel<MODE><<<blocks, 256, 0, s>>>(Wc, d8, F_in, F_out, c, j, joff,
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
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(EQLIN_ERR_CUDA, "cudaGetDevice failed");
  auto kern = spectral8_tc_kernel<MODE>;
  const int smem_max = (int)smem_bytes_for(kMaxFin);
  int maxc = 0;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    DevCache &dc = g_cache[dev];
    if (!dc.attr_set[MODE]) {
      cudaError_t e =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
      if (e != cudaSuccess)
        return set_error(EQLIN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem_max;
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
  CUtensorMap mx, my;
  int rc = make_map_2d(&mx, x, (uint64_t)F_in * 8, (uint64_t)T, (uint64_t)F_in * 16, 64,
                       kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = make_map_2d(&my, y, (uint64_t)F_out * 8, (uint64_t)T, (uint64_t)F_out * 16, 32, 32,
                   CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc) return rc;
  const int64_t bbytes = b_job_offset(MODE, F_in, F_out, num_chunks(F_out), 0);
  BMaps bm;
  for (int k = 0; k < kNumBMaps; ++k) {
    rc = make_map_2d(&bm.m[k], Bpack, 64, (uint64_t)(bbytes / 128), 128, 64, (uint32_t)(4 * (k + 1)),
                     CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
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
  cfg.dynamicSmemBytes = smem_bytes_for(F_in);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mx, my, bm, a);
  if (e != cudaSuccess)
    return set_error(EQLIN_ERR_CUDA, "tensor-core launch: %s", cudaGetErrorString(e));
  return check_launch("spectral8_tc_kernel");
}

}  // namespace

// ---------------------------------------------------------------- interface

bool cyclic_tc_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && N == 8 && tc_shape_ok(kModeCyclic8, Cin, Cout);
}

bool d8_tc_supported(int C, int dtype) {
  return dtype == EQLIN_BF16 && C % 8 == 0 && tc_shape_ok(kModeD8, C / 8, C / 8);
}

size_t cyclic_tc_bytes(int, int Cin, int Cout) {
  return (size_t)b_job_offset(kModeCyclic8, Cin, Cout, num_chunks(Cout), 0);
}

size_t d8_tc_bytes(int C) {
  const int F = C / 8;
  return (size_t)b_job_offset(kModeD8, F, F, num_chunks(F), 0);
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
