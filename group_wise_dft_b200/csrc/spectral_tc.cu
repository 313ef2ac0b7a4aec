// Fused tcgen05 tensor-core path for layers with 8 group slots per field:
// cyclic C_8 EQ-Linear (Flash EQ-Linear, Methodology > Algorithmic Approach:
// real DFT along the group axis, per-bin complex products, inverse DFT) and
// the D8 Fourier-domain linear layer (Quick ViTs review, Key design 2:
// change of basis to irreps, Schur blocks with E shared over its two row
// coordinates, back-transform, GELU in the regular domain).
//
// One persistent kernel does the whole layer; the spectra never leave the SM.
//
//   CTA pair (cluster of 2, tcgen05 cta_group::2, instruction M = 128): each
//   CTA owns 64 token rows of a 128-token tile and holds the tile's whole
//   spectrum as the K-major bf16 A operand (Fin KB, 128-byte swizzle).
//   20 warps per CTA:
//     producer warp    lane k owns weight-ring slot k and streams pre-packed
//                      stages (two 16-field K-slices of every block product
//                      of a 64-output-field chunk) into it; when a slot of a
//                      tile's last chunk is released, the next tile's x for
//                      those block pairs is TMA-loaded into A at once
//     1 MMA issuer     (leader CTA, a converged warp, one elected lane) issues
//                      every MMA of a stage into the double-buffered TMEM
//                      accumulator and commits once to release the slot
//     10 transform     in five groups; rewrite each landed block pair in
//     warps            place (two 128-byte rows per token) as the chunks the
//                      MMA K-steps read
//     8 epilogue       TMEM (16x256b loads) -> inverse 8-point transform
//     warps            (+ GELU) -> 32-byte stores of y
//
// Each MMA K-step reads two adjacent 16-byte chunks of one 128-byte row of A:
//   cyclic: one coordinate over 16 fields; a complex bin takes three real
//           products per K-slice: [Im|Re] += Re X . [Wi;Wr] (N = 2co), then
//           Im += Im X . Wr and Re -= Im X . Wi (negated B)
//   D8:     A1, A2, B1, B2 one coordinate over 16 fields; E two coordinates
//           (b = 0, 1) over 8 fields, rows a = 0, 1 sharing one weight panel
//
// Every wait on an mbarrier is bounded: on timeout the kernel records a code
// in g_fault_state (with this launch's epoch), stops issuing work, lets copies
// in flight land, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "eqlin_internal.cuh"
#include "tc_primitives.cuh"
#include "tc_host.h"
#include "tc_transforms.cuh"
#include "tc_pack_math.cuh"

namespace eqlin {

// [0]: the first code a bounded wait recorded (kept until the host clears it);
// [1]: the epoch of the latest launch whose wait gave up (tc::FaultCtx).
__device__ unsigned int g_fault_state[2] = {0u, 0u};

int read_device_fault(int reset) {
  unsigned int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return -(int)e;
  e = cudaMemcpyFromSymbol(&v, g_fault_state, sizeof v);
  if (e != cudaSuccess) return -(int)e;
  if (reset && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_fault_state, &z, sizeof z);
    if (e != cudaSuccess) return -(int)e;
  }
  return (int)v;
}

unsigned int next_launch_epoch() {
  static std::atomic<unsigned int> counter{0};
  unsigned int e = counter.fetch_add(1u) + 1u;
  if (e == 0u) e = counter.fetch_add(1u) + 1u;   // 0 is never an epoch
  return e;
}

namespace {

// (mode numbers kModeCyclic8, kModeD8, kModeNegacyclic8: tc_pack_math.cuh)
// D8 options (TcArgs::gelu): GELU in the regular domain; input already in
// Fourier coordinates (the forward change of basis is skipped); output in
// Fourier coordinates (with kD8Gelu: Q GELU(Q^T z), the MLP's round trip).
constexpr int kD8Gelu = 1;
constexpr int kD8InFourier = 2;
constexpr int kD8OutFourier = 4;
// Any mode: x already holds coordinates (only placed), and y is fp32 (32 bytes
// per field) instead of the I/O type.
constexpr int kInFourier = kD8InFourier;
constexpr int kOutF32 = 8;
// Negacyclic mode, the odd half of a C_16 layer (its only use, so the
// negacyclic instance always does this): the epilogue reads the even half's
// output ye [T][F_out][8] (TcArgs::y_even) and writes the C_16 output
// y [T][F_out][16] itself: y_g = ye_g + yo_g, y_{g+8} = ye_g - yo_g.
constexpr int kCombine16 = 16;
// negacyclic C_8 (the product modulo z^8 + 1): the odd half of a C_16 layer

// warp roles
constexpr int kThreads = 640;
constexpr int kWarpProd = 0;     // weight-stage producer; TMEM allocation
constexpr int kWarpMma0 = 1;     // MMA issuer
constexpr int kNumIssuers = 1;
constexpr int kDftWarp0 = 2;     // in-place forward transform of x
constexpr int kNumDftWarps = 10;
constexpr int kEpiWarp0 = 12;    // TMEM -> inverse transform -> y
constexpr int kNumEpiWarps = 8;     // two per TMEM lane quarter
static_assert(kEpiWarp0 + kNumEpiWarps == kThreads / 32, "warp roles cover the CTA");

constexpr int kRowsPerCta = 64;
constexpr int kTileTokens = 2 * kRowsPerCta;
constexpr int kBlockBytes = kRowsPerCta * 128;  // one 8-field block of A: 64 rows x 128 B
constexpr int kRingSlotsMax = 8;                // weight ring: as many stages as fit
constexpr int kCtrlBytes = 512;                 // barriers and the TMEM address
constexpr int kSmemLimit = 232448;              // opt-in shared memory per CTA
constexpr int kCoMax = 64;                      // output fields per chunk
constexpr int kBRow = 512;                      // TMA row of the packed weights (bytes): a
                                                // stage is a few long rows, not many 128-byte ones
constexpr int kMaxFin = 160;                    // A operand = Fin KB of shared memory
constexpr int kMaxBlocks = kMaxFin / 8;
constexpr int kMaxPairs = kMaxBlocks / 2;       // block pairs = weight stages per chunk
constexpr int kDftWarpsPerGroup = 2;            // one group transforms 64 token rows
constexpr int kDftGroups = kNumDftWarps / kDftWarpsPerGroup;    // 5
// In the cyclic C_8 and p4 modes, block pairs kDftGroups .. kDftGroups +
// kEpiHelpGroups - 1 of every tile are transformed by the epilogue warps (as
// four more two-warp groups): at a tile boundary they are free (the last
// chunk's epilogue can wait until the next tile's first chunk runs), so all but
// one of the tile's block pairs are transformed in one round instead of two.
// Not in the D8 mode, whose epilogue (back-transform and GELU of every output)
// is its busiest role, nor in the negacyclic mode, whose epilogue also reads
// the even half's outputs and writes twice the bytes.
constexpr int kEpiHelpGroups = kNumEpiWarps / kDftWarpsPerGroup;  // 4
template <int MODE>
__host__ __device__ constexpr bool epilogue_helps() { return MODE == kModeCyclic8 || MODE == kModeCyclic4; }
// In the D8 and negacyclic modes it is the other way round: the epilogue
// (back-transform and GELU of every output; or, for the odd half of C_16, the
// even half's outputs read and twice the bytes written) paces the layer, and
// transform warps 0..7 (two per TMEM lane quarter, as the epilogue warps) take
// every other 8-column group of each chunk's epilogue; they transform the next
// tile's block pairs before their share of a tile's last chunk.
constexpr int kD8HelpWarps = 8;
template <int MODE>
__host__ __device__ constexpr bool transform_warps_help_epilogue() {
  return MODE == kModeD8 || MODE == kModeNegacyclic8;
}
template <int MODE>
__host__ __device__ constexpr int epilogue_warps() {
  return kNumEpiWarps + (transform_warps_help_epilogue<MODE>() ? kD8HelpWarps : 0);
}
// Which two-warp group transforms block pair jp: with epilogue help, the
// transform groups take jp < kDftGroups and the pairs after the helped ones
// (from group 0 on, which finishes its first pair earliest) and the epilogue
// groups the rest; without, transform group jp mod kDftGroups.
template <int MODE>
__host__ __device__ constexpr bool pair_by_epilogue(int jp) {
  return epilogue_helps<MODE>() && jp >= kDftGroups && jp < kDftGroups + kEpiHelpGroups;
}
template <int MODE>
__host__ __device__ constexpr int pair_group(int jp) {
  if (!epilogue_helps<MODE>()) return jp % kDftGroups;
  return jp < kDftGroups ? jp
                         : (pair_by_epilogue<MODE>(jp) ? jp - kDftGroups : (jp - kEpiHelpGroups) % kDftGroups);
}
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccBufCols = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kSleepNs = 128;              // back-off of warps that wait for long phases

__host__ __device__ inline int chunk_fields(int F_out, int c) {
  const int r = F_out - c * kCoMax;
  return r < kCoMax ? r : kCoMax;
}
__host__ __device__ inline int num_chunks(int F_out) { return (F_out + kCoMax - 1) / kCoMax; }

// A weight stage is one 16-field K-slice (block pair jp) of every block
// product of a chunk of `co` output fields, per CTA half (hc = co/2 output
// fields).  Panels, in order:
//   cyclic: Re X0, Re X4, then the complex bins 1, 2, 3
//   D8:     A1, A2, B1, B2, then E for K-step 2jp and 2jp+1
// Cyclic real and D8 1-D panels: [K-chunk 2][hc rows][8 bf16] (16*co bytes),
// the K-chunks being the 8 fields of blocks 2jp and 2jp+1.
// Cyclic complex bin panel: [K-chunk 2][co rows: Wi of the hc fields, then Wr
// of the hc fields][8] (32*co bytes).
// D8 E panel: [K-chunk = b 2][co rows = (b', field)][8 fields] (32*co bytes).
// A complex bin takes three MMAs per K-slice:
//   [Im Y | Re Y] += Re X . [Wi ; Wr]   (one MMA over all co rows, N = 2co)
//   Im Y += Im X . Wr                   (the Wr rows)
//   Re Y -= Im X . Wi                   (the Wi rows, the instruction's negate-B bit)
// so Wr and Wi are stored once each and Re X is read from shared memory once
// for both outputs.  These MMAs (64 token rows per CTA) are bound by their
// shared-memory operand reads, not by tensor math: an MMA costs about
// (A bytes + this CTA's B bytes) / 128 cycles, so reading an A chunk once for
// N = 2co columns instead of twice for co is the cheaper form.
// Negacyclic: four complex bins, each a combined [Wi; Wr] panel as above.
__host__ __device__ inline int num_panels(int mode) {
  return mode == kModeCyclic8 ? 5 : (mode == kModeNegacyclic8 ? 4 : 6);
}
// C_4: per row r of the block pair, panels 3r..3r+2 = W0, W2 (real), bin 1 as [Wi; Wr]
__host__ __device__ inline int panel_bytes(int mode, int k, int co) {
  if (mode == kModeCyclic8) return k < 2 ? 16 * co : 32 * co;
  if (mode == kModeNegacyclic8) return 32 * co;
  if (mode == kModeCyclic4) return k % 3 < 2 ? 16 * co : 32 * co;
  return k < 4 ? 16 * co : 32 * co;
}
// B rows per K-chunk of panel k (its leading byte offset is 16 bytes per row).
__host__ __device__ inline int panel_rows(int mode, int k, int co) { return panel_bytes(mode, k, co) / 32; }
__host__ __device__ inline int panel_offset(int mode, int k, int co) {
  int off = 0;
  for (int i = 0; i < k; ++i) off += panel_bytes(mode, i, co);
  return off;
}
__host__ __device__ inline int stage_bytes(int mode, int co) {
  return panel_offset(mode, num_panels(mode), co);
}
#ifndef EQLIN_KS_FULL
#define EQLIN_KS_FULL 2
#endif
// K-slices (block pairs) per ring stage of chunk c: kKsFull for a full chunk,
// twice that for a narrow last chunk (at most half of kCoMax output fields),
// halved while it does not divide the K-slices.  Every stage costs the issuer
// a fixed loop overhead (wait, commit, bookkeeping), so fewer, larger stages
// leave more of its time to the MMAs themselves.
constexpr int kKsFull = EQLIN_KS_FULL;
__host__ __device__ inline int chunk_ks(int F_in, int F_out, int c) {
  const int nst = F_in / 16;
  int ks = 2 * chunk_fields(F_out, c) <= kCoMax ? 2 * kKsFull : kKsFull;
  while (ks > 1 && nst % ks != 0) ks /= 2;
  return ks;
}
// Bytes of one CTA half of a ring stage of chunk c.
__host__ __device__ inline int chunk_stage_bytes(int mode, int F_in, int F_out, int c) {
  return chunk_ks(F_in, F_out, c) * stage_bytes(mode, chunk_fields(F_out, c));
}
// Byte offset of the panels of (chunk c, K-slice jp, CTA half h).  A ring
// stage s of chunk c holds K-slices s*ks .. s*ks+ks-1 (ks = chunk_ks) and its
// two CTA halves are contiguous: [h = 0: slices][h = 1: slices].
__host__ __device__ inline int64_t stage_offset(int mode, int F_in, int F_out, int c, int jp, int h) {
  const int64_t full = (int64_t)2 * (F_in / 16) * stage_bytes(mode, kCoMax);
  const int ks = chunk_ks(F_in, F_out, c);
  const int s = jp / ks, q = jp - s * ks;
  return (int64_t)c * full + (int64_t)((2 * s + h) * ks + q) * stage_bytes(mode, chunk_fields(F_out, c));
}
__host__ __device__ inline int64_t packed_bytes(int mode, int F_in, int F_out) {
  return stage_offset(mode, F_in, F_out, num_chunks(F_out) - 1, F_in / 16, 0);
}

// One MMA of an issuer's stage: A block (2*jp + blk) and chunk pair `pair`,
// weight panel `panel` starting at row roff * co/2, TMEM column group
// `dgroup`, B rows per CTA co (wide = 1: N = 2co, column groups dgroup and
// dgroup + 1) or co/2 (N = co), negated B.
struct MmaDesc {
  int blk, pair, panel, dgroup, wide, neg, roff;
};
constexpr int kMmaLists = 4;
constexpr int kMaxMmaPerList = 3;
// A stage's MMAs are the lists i = 0..3 of mma_desc(mode, i, m), m < mma_count(mode, i),
// in order; the lists write disjoint TMEM column groups.
__host__ __device__ constexpr int mma_count(int mode, int i) {
  if (mode == kModeCyclic8) return i == 3 ? 2 : 3;
  if (mode == kModeNegacyclic8) return 3;
  if (mode == kModeCyclic4) return i % 2 == 0 ? 2 : 3;
  return 2;
}
__host__ __device__ constexpr MmaDesc mma_desc(int mode, int i, int m) {
  if (mode == kModeCyclic8) {
    // A coordinate c (as in fwd_cyclic8) sits in block c/4, chunk pair c%4;
    // column groups as in group_coord.  Issuer b-1 owns complex bin b (panel
    // b+1, groups Im = 2b, Re = 2b+1); issuer 3 the real bins 0 and 4.
    // (a switch rather than an indexed table keeps it out of local memory)
    switch (i * 4 + m) {
      case 0: return {0, 1, 2, 2, 1, 0, 0};   // [Im|Re] Y1 += Re X1 . [Wi;Wr]
      case 1: return {0, 2, 2, 2, 0, 0, 1};   // Im Y1 += Im X1 . Wr
      case 2: return {0, 2, 2, 3, 0, 1, 0};   // Re Y1 -= Im X1 . Wi
      case 4: return {0, 3, 3, 4, 1, 0, 0};   // bin 2: Re X2 = c3, Im X2 = c4
      case 5: return {1, 0, 3, 4, 0, 0, 1};
      case 6: return {1, 0, 3, 5, 0, 1, 0};
      case 8: return {1, 1, 4, 6, 1, 0, 0};   // bin 3: Re X3 = c5, Im X3 = c6
      case 9: return {1, 2, 4, 6, 0, 0, 1};
      case 10: return {1, 2, 4, 7, 0, 1, 0};
      case 12: return {0, 0, 0, 0, 0, 0, 0};  // Re Y0 += Re X0 . W0
      case 13: return {1, 3, 1, 1, 0, 0, 0};  // Re Y4 += Re X4 . W4 (Re X4 = c7)
      default: return {0, 0, 0, 0, 0, 0, 0};
    }
  }
  if (mode == kModeNegacyclic8) {
    // Bin b = i: Re D_b is coordinate 2b, Im D_b is 2b + 1 (as in
    // fwd_negacyclic8; block c/4, chunk pair c%4); panel b holds [Wi; Wr];
    // column groups Im Y_b = 2b, Re Y_b = 2b + 1.
    switch (i * 4 + m) {
      case 0: return {0, 0, 0, 0, 1, 0, 0};   // [Im|Re] Y0 += Re D0 . [Wi;Wr]
      case 1: return {0, 1, 0, 0, 0, 0, 1};   // Im Y0 += Im D0 . Wr
      case 2: return {0, 1, 0, 1, 0, 1, 0};   // Re Y0 -= Im D0 . Wi
      case 4: return {0, 2, 1, 2, 1, 0, 0};   // bin 1: Re D1 = c2, Im D1 = c3
      case 5: return {0, 3, 1, 2, 0, 0, 1};
      case 6: return {0, 3, 1, 3, 0, 1, 0};
      case 8: return {1, 0, 2, 4, 1, 0, 0};   // bin 2: Re D2 = c4, Im D2 = c5
      case 9: return {1, 1, 2, 4, 0, 0, 1};
      case 10: return {1, 1, 2, 5, 0, 1, 0};
      case 12: return {1, 2, 3, 6, 1, 0, 0};  // bin 3: Re D3 = c6, Im D3 = c7
      case 13: return {1, 3, 3, 6, 0, 0, 1};
      case 14: return {1, 3, 3, 7, 0, 1, 0};
      default: return {0, 0, 0, 0, 0, 0, 0};
    }
  }
  if (mode == kModeCyclic4) {
    // Row r = i / 2 of the block pair holds 16 C_4 fields, coordinate q
    // ([Re X0, Re X1, Im X1, Re X2]) in chunk pair q; panels 3r (W0), 3r + 1
    // (W2), 3r + 2 (bin 1 as [Wi; Wr]); column groups Re Y0 = 0, Im Y1 = 1,
    // Re Y1 = 2, Re Y2 = 3.
    switch (i * 4 + m) {
      case 0: return {0, 0, 0, 0, 0, 0, 0};   // Re Y0 += Re X0 . W0          (row 0)
      case 1: return {0, 3, 1, 3, 0, 0, 0};   // Re Y2 += Re X2 . W2
      case 4: return {0, 1, 2, 1, 1, 0, 0};   // [Im|Re] Y1 += Re X1 . [Wi;Wr]
      case 5: return {0, 2, 2, 1, 0, 0, 1};   // Im Y1 += Im X1 . Wr
      case 6: return {0, 2, 2, 2, 0, 1, 0};   // Re Y1 -= Im X1 . Wi
      case 8: return {1, 0, 3, 0, 0, 0, 0};   // the same for row 1
      case 9: return {1, 3, 4, 3, 0, 0, 0};
      case 12: return {1, 1, 5, 1, 1, 0, 0};
      case 13: return {1, 2, 5, 1, 0, 0, 1};
      case 14: return {1, 2, 5, 2, 0, 1, 0};
      default: return {0, 0, 0, 0, 0, 0, 0};
    }
  }
  switch (i) {
    case 0: return m == 0 ? MmaDesc{0, 0, 0, 0, 0, 0, 0} : MmaDesc{0, 1, 1, 1, 0, 0, 0};    // A1 | A2
    case 1: return m == 0 ? MmaDesc{1, 0, 2, 2, 0, 0, 0} : MmaDesc{1, 1, 3, 3, 0, 0, 0};    // B1 | B2
    case 2: return MmaDesc{m, 2, 4 + m, 4, 1, 0, 0};                                       // E row a = 0
    default: return MmaDesc{m, 3, 4 + m, 6, 1, 0, 0};                                      // E row a = 1
  }
}

// Coordinate held by TMEM column group k (k = 0..7) of an accumulator buffer:
// cyclic [Re Y0, Re Y4, Im Y1, Re Y1, Im Y2, Re Y2, Im Y3, Re Y3] (the complex
// bins' rows are ordered [Im; Re]); D8 in coordinate order.
__host__ __device__ inline int group_coord(int mode, int k) {
  if (mode == kModeCyclic8) {
    const int map[8] = {0, 7, 2, 1, 4, 3, 6, 5};
    return map[k];
  }
  if (mode == kModeNegacyclic8) return k ^ 1;   // [Im Y0, Re Y0, Im Y1, Re Y1, ..]
  if (mode == kModeCyclic4) {                   // [Re Y0, Im Y1, Re Y1, Re Y2] -> coordinate
    const int map[4] = {0, 2, 1, 3};
    return map[k & 3];
  }
  return k;
}

bool tc_shape_ok(int F_in, int F_out) {
  return F_in >= 16 && F_in <= kMaxFin && F_in % 16 == 0 && F_out >= 32 && F_out % 32 == 0;
}

// Ring slot size (the largest stage) and how many slots fit next to A.
struct RingShape {
  int slot_bytes, nslots;
};
RingShape ring_shape(int mode, int F_in, int F_out) {
  RingShape r;
  const int a = chunk_stage_bytes(mode, F_in, F_out, 0);
  const int b = chunk_stage_bytes(mode, F_in, F_out, num_chunks(F_out) - 1);
  r.slot_bytes = a > b ? a : b;
  const int room = kSmemLimit - 1024 - F_in * 1024 - kCtrlBytes;
  r.nslots = room / r.slot_bytes;
  if (r.nslots > kRingSlotsMax) r.nslots = kRingSlotsMax;
  return r;
}

size_t smem_bytes_for(int F_in, const RingShape &r) {
  return 1024 + (size_t)F_in * 1024 + (size_t)r.nslots * r.slot_bytes + kCtrlBytes;
}

// ---------------------------------------------------------------- transforms
// (paired fp32 helpers, the forward C_8 transform and bf16 packing: tc_transforms.cuh)

// (inverse C_8, negacyclic, D8 transforms and GELU: tc_transforms.cuh)

// Where coordinate c of block q_b (b = 0: block 2jp, 1: block 2jp+1) goes:
// row (0: block 2jp's 128-byte row, 1: block 2jp+1's) and 16-byte chunk.
template <int MODE>
__host__ __device__ __forceinline__ constexpr void a_place(int c, int b, int &row, int &chunk) {
  if (MODE == kModeCyclic8 || MODE == kModeNegacyclic8) {
    row = c >> 2;
    chunk = 2 * (c & 3) + b;
  } else if (MODE == kModeCyclic4) {
    // coordinate c % 4 of the first (c < 4) or second C_4 field of each of the
    // row's 8 super-fields: chunk pair c % 4 holds coordinate c % 4 of all 16
    // fields, the even fields in its first chunk and the odd in its second
    row = b;
    chunk = 2 * (c & 3) + (c >> 2);
  } else if (c < 4) {          // A1, A2 -> row 0; B1, B2 -> row 1
    row = c >> 1;
    chunk = 2 * (c & 1) + b;
  } else {                     // E: the block's own row, chunks 4..7
    row = b;
    chunk = c;
  }
}

// One thread per token: transform both blocks of the pair in place.  Block 0
// (row 0) is read whole and transformed; before its outputs are written, the
// chunks of row 1 that they overwrite are read; then the rest of row 1 is read
// and block 1 is transformed.  At most 32 + 16 payload registers are live, so
// the transform does not spill.
template <int MODE, bool H>
__device__ __forceinline__ void transform_block(const uint4 (&in)[8], uint32_t (&out)[8][4], int flags) {
#pragma unroll
  for (int fp = 0; fp < 4; ++fp) {
    float2 x[8], z[8];
    unpack_x8_pair<H>(in[2 * fp], in[2 * fp + 1], x);
    if (flags & kInFourier) {   // already coordinates: only placed
#pragma unroll
      for (int c = 0; c < 8; ++c) z[c] = x[c];
    } else if (MODE == kModeCyclic8)
      fwd_cyclic8(x, z);
    else if (MODE == kModeNegacyclic8)
      fwd_negacyclic8(x, z);
    else if (MODE == kModeCyclic4)
      fwd_cyclic4x2(x, z);
    else
      fwd_d8(x, z);
#pragma unroll
    for (int c = 0; c < 8; ++c) out[c][fp] = pack_x2<H>(z[c].x, z[c].y);
  }
}

// Whether block 0's output coordinates overwrite chunk `ch` of row 1.
template <int MODE>
__device__ __forceinline__ constexpr bool row1_chunk_taken_by_block0(int ch) {
  bool taken = false;
  for (int c = 0; c < 8; ++c) {
    int row = 0, chunk = 0;
    a_place<MODE>(c, 0, row, chunk);
    if (row == 1 && chunk == ch) taken = true;
  }
  return taken;
}

template <int MODE, bool H>
__device__ __forceinline__ void transform_rows(uint8_t *row0, uint8_t *row1, int sw, int flags) {
  uint4 in[8];
  uint32_t out[8][4];
#pragma unroll
  for (int f = 0; f < 8; ++f) in[f] = *reinterpret_cast<const uint4 *>(row0 + ((f ^ sw) << 4));
  transform_block<MODE, H>(in, out, flags);
#pragma unroll
  for (int f = 0; f < 8; ++f)
    if (row1_chunk_taken_by_block0<MODE>(f))
      in[f] = *reinterpret_cast<const uint4 *>(row1 + ((f ^ sw) << 4));
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    int row, chunk;
    a_place<MODE>(c, 0, row, chunk);
    *reinterpret_cast<uint4 *>((row ? row1 : row0) + ((chunk ^ sw) << 4)) =
        make_uint4(out[c][0], out[c][1], out[c][2], out[c][3]);
  }
#pragma unroll
  for (int f = 0; f < 8; ++f)
    if (!row1_chunk_taken_by_block0<MODE>(f))
      in[f] = *reinterpret_cast<const uint4 *>(row1 + ((f ^ sw) << 4));
  transform_block<MODE, H>(in, out, flags);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    int row, chunk;
    a_place<MODE>(c, 1, row, chunk);
    *reinterpret_cast<uint4 *>((row ? row1 : row0) + ((chunk ^ sw) << 4)) =
        make_uint4(out[c][0], out[c][1], out[c][2], out[c][3]);
  }
}


// One 8-column group (fg) of the negacyclic (C_16 odd half) epilogue for one
// warp: the even half's outputs of the thread's 4 items (loaded first, so the
// global and TMEM load latencies overlap), TMEM rows tb.., the inverse
// negacyclic transform, and the C_16 outputs y_g = ye_g + yo_g,
// y_{g+8} = ye_g - yo_g as 64-byte runs (the odd half's output never reaches
// memory).  Items as in the epilogue role (2 fields x 2 tokens per thread).
// Not inlined: its registers then stay out of the loops that call it.
__device__ __noinline__ void neg16_epilogue_group(uint32_t tb, int fg, int half, int64_t tok0,
                                                     int field_base, int64_t T, int F_out, uint8_t *ybase,
                                                     const void *y_even) {
  using namespace tc;
  uint4 ye[2][2];
#pragma unroll
  for (int r8 = 0; r8 < 2; ++r8) {
    const int64_t tok = tok0 + 8 * r8;
    const uint4 *src = reinterpret_cast<const uint4 *>(y_even) + (size_t)(tok < T ? tok : 0) * F_out +
                       field_base + fg;
    ye[r8][0] = __ldcs(src);
    ye[r8][1] = __ldcs(src + 1);
  }
  uint32_t v[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) tmem_ld_16x256b(tb + (uint32_t)(kk * half + fg), v[kk]);
  tmem_wait_ld();
#pragma unroll
  for (int ip = 0; ip < 4; ip += 2) {     // items ip, ip + 1 as the two float2 lanes
    float2 z[8], yv[8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      z[group_coord(kModeNegacyclic8, kk)] =
          make_float2(__uint_as_float(v[kk][ip]), __uint_as_float(v[kk][ip + 1]));
    inv_negacyclic8(z, yv);
    // items ip, ip + 1: token tok0 + 8 (ip / 2), fields f, f + 1, whose even-half
    // outputs are 32 contiguous bytes of ye and whose C_16 outputs are 64
    // contiguous bytes of y
    const int64_t tok = tok0 + 8 * (ip >> 1);
    if (tok < T) {
      const size_t item = (size_t)tok * F_out + field_base + fg;
      float2 ev[8];
      unpack_x8_pair<false>(ye[ip >> 1][0], ye[ip >> 1][1], ev);   // ev[g] = (ye_g of f, of f + 1)
      uint32_t lo0[4], hi0[4], lo1[4], hi1[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 a = ev[2 * q], b = ev[2 * q + 1], ya = yv[2 * q], yb = yv[2 * q + 1];
        lo0[q] = pack_x2<false>(a.x + ya.x, b.x + yb.x);
        hi0[q] = pack_x2<false>(a.x - ya.x, b.x - yb.x);
        lo1[q] = pack_x2<false>(a.y + ya.y, b.y + yb.y);
        hi1[q] = pack_x2<false>(a.y - ya.y, b.y - yb.y);
      }
      uint8_t *dst = ybase + item * 32;
      st_global_v8(dst, lo0, hi0);
      st_global_v8(dst + 32, lo1, hi1);
    }
  }
}

// One 8-column group (fg) of a D8 chunk's epilogue for one warp: TMEM rows
// tb.., items as in the epilogue role (2 fields x 2 tokens per thread), the
// back-transform (and GELU, or the round trip back to coordinates, or the
// coordinates as they are) and 32-byte stores of y.
template <bool H>
__device__ __forceinline__ void d8_epilogue_group(uint32_t tb, int fg, int half, int64_t tok0, int field_base,
                                                  int64_t T, int F_out, uint8_t *ybase, int flags) {
  using namespace tc;
  uint32_t v[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) tmem_ld_16x256b(tb + (uint32_t)(kk * half + fg), v[kk]);
  tmem_wait_ld();
  uint32_t w[4][4];
#pragma unroll
  for (int ip = 0; ip < 4; ip += 2) {     // items ip, ip + 1 as the two float2 lanes
    float2 z[8], yv[8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      z[kk] = make_float2(__uint_as_float(v[kk][ip]), __uint_as_float(v[kk][ip + 1]));
    if ((flags & (kD8OutFourier | kD8Gelu)) == kD8OutFourier) {
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) yv[gg] = z[gg];   // coordinates out as they are
    } else {
      inv_d8(z, yv);
      if (flags & kD8Gelu) {
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) yv[gg] = gelu_tanh2(yv[gg]);
      }
      if (flags & kD8OutFourier) {   // the GELU round trip: back to coordinates
        float2 zz[8];
        fwd_d8(yv, zz);
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) yv[gg] = zz[gg];
      }
    }
#pragma unroll
    for (int p2 = 0; p2 < 4; ++p2) {
      w[ip][p2] = pack_x2<H>(yv[2 * p2].x, yv[2 * p2 + 1].x);
      w[ip + 1][p2] = pack_x2<H>(yv[2 * p2].y, yv[2 * p2 + 1].y);
    }
  }
  // items 0, 1: token tok0, fields f, f+1; items 2, 3: token tok0 + 8
#pragma unroll
  for (int r8 = 0; r8 < 2; ++r8) {
    const int64_t tok = tok0 + 8 * r8;
    if (tok < T) st_global_v8(ybase + (tok * F_out + field_base + fg) * 16, w[2 * r8], w[2 * r8 + 1]);
  }
}

// Report a transformed block pair to the issuer (the leader CTA's a_full
// barrier).  The leader's own warps arrive with a CTA-scope release, which is
// all the issuer (in the same CTA) needs; the peer's warps need a cluster-scope
// release, which blocks the arriving warp for the better part of a
// microsecond (traces), so the leader's warps are spared it (C_8, 160 x 160
// fields, T = 131072: about 2 % faster).
__device__ __forceinline__ void arrive_a_full(uint32_t leader_bar_cluster) {
  if (tc::cluster_ctarank() == 0)
    tc::mbar_arrive_cluster_cta(leader_bar_cluster);
  else
    tc::mbar_arrive_cluster(leader_bar_cluster);
}

// The epilogue warps' share of the forward transform, as a call: its
// registers are then not allocated across the whole epilogue loop.
template <int MODE, bool H>
__device__ __noinline__ bool transform_pair_call(uint8_t *pair_base, uint32_t bar_x, uint32_t parity,
                                                 tc::FaultCtxSmem fault, int row, int flags,
                                                 uint32_t a_full_cluster) {
  using namespace tc;
  if (!mbar_wait_bounded(bar_x, parity, fault, FAULT_WAIT_X_FULL, kWaitLimitNs, kSleepNs)) return false;
  uint8_t *r0 = pair_base + row * 128;
  transform_rows<MODE, H>(r0, r0 + kBlockBytes, row & 7, flags);
  fence_proxy_async_smem();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) arrive_a_full(a_full_cluster);
  return true;
}

// ---------------------------------------------------------------- kernel

struct TcArgs {
  void *y;          // [T][F_out][8] bf16, 32-byte aligned
  int64_t T;
  int F_in;
  int F_out;
  int ntiles;
  int gelu;         // option flags: kD8Gelu | kD8InFourier | kD8OutFourier | kOutF32 | kCombine16
  const void *y_even;   // kCombine16: the even half's output ye [T][F_out][8] bf16
  int nslots;       // weight ring slots
  int slot_bytes;   // bytes per slot (the largest stage)
  unsigned int epoch;   // this launch's fault epoch (next_launch_epoch)
};

template <int MODE, bool H>
__global__ void __launch_bounds__(kThreads, 1)
    spectral8_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_b_full,
                        const __grid_constant__ CUtensorMap map_b_last, const TcArgs args) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);

  const int F_in = args.F_in;
  const int F_out = args.F_out;
  const int nchunks = num_chunks(F_out);
  const int nstage = F_in / 16; // weight stages (block pairs) per chunk

  const uint32_t sA = base;
  const uint32_t sB = sA + (uint32_t)F_in * 1024u;
  const int nslots = args.nslots;
  const uint32_t slot_bytes = (uint32_t)args.slot_bytes;
  const uint32_t sBar = sB + (uint32_t)nslots * slot_bytes;
  // x_full[jp]: block pair jp of x landed (this CTA); a_full[jp]: block pair
  // jp transformed in both CTAs (leader's copy is the one used)
  auto bar_x_full = [&](int jp) { return sBar + 8u * jp; };                     // kMaxPairs
  auto bar_a_full = [&](int jp) { return sBar + 8u * (kMaxPairs + jp); };       // kMaxPairs
  auto bar_b_full = [&](int i) { return sBar + 8u * (2 * kMaxPairs + i); };     // kRingSlotsMax
  auto bar_b_empty = [&](int i) { return sBar + 8u * (2 * kMaxPairs + kRingSlotsMax + i); };
  auto bar_acc_full = [&](int i) { return sBar + 8u * (2 * kMaxPairs + 2 * kRingSlotsMax + i); };
  auto bar_acc_empty = [&](int i) {
    return sBar + 8u * (2 * kMaxPairs + 2 * kRingSlotsMax + 2 + i);
  };
  const uint32_t tmem_slot = sBar + 8u * (2 * kMaxPairs + 2 * kRingSlotsMax + 4);
  static_assert(8 * (2 * kMaxPairs + 2 * kRingSlotsMax + 4) + 8 <= kCtrlBytes, "control block");
  volatile uint32_t *tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t *>(gbase + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  // the launch's epoch sits in the control block (written below), so no
  // register holds it across the kernel
  const uint32_t epoch_slot = tmem_slot + 4u;
  const FaultCtxSmem fault{g_fault_state, epoch_slot};

  if (threadIdx.x == 0) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(epoch_slot), "r"(args.epoch) : "memory");
    for (int jp = 0; jp < kMaxPairs; ++jp) {
      mbar_init(bar_x_full(jp), 1);
      mbar_init(bar_a_full(jp), 2 * kDftWarpsPerGroup);   // the group's warps in both CTAs
    }
    for (int i = 0; i < kRingSlotsMax; ++i) {
      mbar_init(bar_b_full(i), 1);
      mbar_init(bar_b_empty(i), kNumIssuers);        // every issuer releases every stage
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc_full(i), kNumIssuers);
      mbar_init(bar_acc_empty(i), 2 * epilogue_warps<MODE>());   // every epilogue warp of both CTAs
    }
    fence_mbarrier_init_cluster();
  }
  if (warp == kWarpProd) tmem_alloc_pair(tmem_slot, kTmemCols);
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  tcgen05_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  const int ntile_local = args.ntiles > pair ? (args.ntiles - pair + npairs - 1) / npairs : 0;
  const int total_chunks = ntile_local * nchunks;  // global chunk index g = tile_iter * nchunks + c

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    // Lane k owns ring slot k and loads the stages st = k, k + S, k + 2S, ...
    // (S = the number of ring slots), so the slots refill in parallel: one thread's
    // bookkeeping and TMA issue latency would otherwise sit on the ring's
    // critical path once per stage.
    //
    // The release of a slot (every issuer's commit after the stage's MMAs)
    // also means those MMAs are done with the stage's A block pair; when the
    // released stage belongs to a tile's last chunk, that block pair is free
    // and the next tile's x for it is loaded at once, so the next tile's
    // loads and transforms overlap this tile's remaining MMAs.
    if (lane == 0) {
      prefetch_tensormap(&map_b_full);
      prefetch_tensormap(&map_b_last);
      prefetch_tensormap(&map_x);
    }
    const uint32_t leader_b_full0 = mapa_shared(bar_b_full(0), 0);
    auto load_x = [&](int ti, int jp) {
      const int row0 = (pair + ti * npairs) * kTileTokens + (int)rank * kRowsPerCta;
      mbar_arrive_expect_tx(bar_x_full(jp), 2u * kBlockBytes);
      tma_load_2d(sA + (uint32_t)(2 * jp) * kBlockBytes, &map_x, bar_x_full(jp), 2 * jp * 64, row0);
      tma_load_2d(sA + (uint32_t)(2 * jp + 1) * kBlockBytes, &map_x, bar_x_full(jp),
                  (2 * jp + 1) * 64, row0);
    };
    if (ntile_local > 0 && lane < nstage) load_x(0, lane);
    const int rows_full = chunk_stage_bytes(MODE, F_in, F_out, 0) / kBRow;
    const int rows_last = chunk_stage_bytes(MODE, F_in, F_out, nchunks - 1) / kBRow;
    const int chunk_stride = 2 * nstage * (stage_bytes(MODE, kCoMax) / kBRow);
    const uint32_t tx_full = 2u * kBRow * (uint32_t)rows_full;
    const uint32_t tx_last = 2u * kBRow * (uint32_t)rows_last;
    const int ks_last = chunk_ks(F_in, F_out, nchunks - 1);
    const int ns_full = nstage / chunk_ks(F_in, F_out, 0);   // ring stages of a full chunk
    const int lead = (nchunks - 1) * ns_full;         // stages of the full chunks
    const int per_tile = lead + nstage / ks_last;     // ring stages per tile
    const int total = ntile_local * per_tile;
    const bool owner = lane < nslots;
    const uint32_t my_empty = bar_b_empty(owner ? lane : 0);
    const uint32_t my_slot = sB + (uint32_t)(owner ? lane : 0) * slot_bytes;
    const uint32_t my_full = leader_b_full0 + 8u * (uint32_t)(owner ? lane : 0);
    int p_tl = -1, p_c = 0, p_s = 0;           // this lane's previous stage
    uint32_t ph = 0;
    bool ok = true;
    for (int st = lane; ok; st += nslots) {
      const bool has_cur = owner && st < total;
      const bool has_prev = owner && st - nslots >= 0 && st - nslots < total;
      if (!__any_sync(0xffffffffu, has_cur || has_prev)) break;
      int tl = 0, c = 0, s = 0, rem = 0, q_lo = 0, q_hi = 0;
      if (has_cur) {
        tl = st / per_tile;
        rem = st - tl * per_tile;
        c = rem < lead ? rem / ns_full : nchunks - 1;
        s = rem - c * ns_full;
        // block pairs of the next tile's x to pull into L2 at this stage
        q_lo = (rem * nstage + per_tile - 1) / per_tile;
        q_hi = ((rem + 1) * nstage + per_tile - 1) / per_tile;
      }
      // wait for this slot's previous stage to be released (a fresh slot
      // passes at once), then refill it; every lane polls its own slot
      bool done = !(has_cur || has_prev);
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t it = 1; !__all_sync(0xffffffffu, done); ++it) {
        const bool ready = !done && mbar_test_wait(my_empty, ph ^ 1u);
        // back off while no slot is ready: the issuer sharing this
        // scheduler needs the issue slots
        if (!__any_sync(0xffffffffu, ready)) __nanosleep(32);
        if (ready) {
          // most urgent first: this stage's weights, then the next tile's x
          // for the block pairs the released stage freed, then L2 prefetches
          if (has_cur) {
            const bool last = c == nchunks - 1;
            const int rows_c = last ? rows_last : rows_full;
            const int row = c * chunk_stride + ((int)rank + 2 * s) * rows_c;
            if (leader) mbar_arrive_expect_tx(my_full, last ? tx_last : tx_full);
            tma_load_2d_pair(my_slot, last ? &map_b_last : &map_b_full, my_full, 0, row);
          }
          if (has_prev && p_c == nchunks - 1 && p_tl + 1 < ntile_local)
            for (int q = 0; q < ks_last; ++q) load_x(p_tl + 1, p_s * ks_last + q);
          // pull the next tile's x into L2 while this tile runs, block pairs
          // spread evenly over the tile's stages so the DRAM reads spread
          // too: its load, issued when the last chunk frees the block pair,
          // then hits L2
          if (has_cur && tl + 1 < ntile_local) {
            const int row_n = (pair + (tl + 1) * npairs) * kTileTokens + (int)rank * kRowsPerCta;
            for (int q = q_lo; q < q_hi; ++q) {
              tma_prefetch_2d(&map_x, 2 * q * 64, row_n);
              tma_prefetch_2d(&map_x, (2 * q + 1) * 64, row_n);
            }
          }
          done = true;
        }
        if ((it & 63u) == 0) {
          // the fault word is read only once this wait for the slots has lasted long (a
          // global load here would stall the whole producer warp)
          const uint64_t waited = globaltimer_ns() - t0;
          bool give_up = waited > kFaultCheckAfterNs && fault_raised(fault);
          if (!done && waited > kWaitLimitNs) {
            fault_raise(fault, (unsigned int)FAULT_WAIT_B_EMPTY);
            give_up = true;
          }
          if (__any_sync(0xffffffffu, give_up)) {
            ok = false;
            break;
          }
        }
      }
      p_tl = has_cur ? tl : -1;
      p_c = c;
      p_s = s;
      ph ^= 1u;
    }
  } else if (warp == kWarpMma0) {
    // ------------------------------------------------------------ MMA issue (leader CTA)
    // One converged warp; one elected lane issues every MMA of a stage and
    // commits once.  A single issuer keeps the tensor pipe fed at its own rate
    // (measured: a stage's 14 N=64 MMAs take the pipe's ~350 cycles), where
    // several issuers meeting at every stage's barrier left it idle between
    // stages.  Descriptors are kept as their low 32-bit words (start address
    // and leading byte offset); a stage only adds the slot and K-slice offsets.
    if (leader) {
      constexpr int NM = MODE == kModeCyclic8 ? 11 : (MODE == kModeNegacyclic8 ? 12 : (MODE == kModeCyclic4 ? 10 : 8));
      MmaDesc md[NM];
      uint32_t acc_first[NM];   // 1: an earlier MMA of the stage already wrote the group
      {
        int f = 0;
#pragma unroll
        for (int i = 0; i < kMmaLists; ++i)
#pragma unroll
          for (int m = 0; m < kMaxMmaPerList; ++m)
            if (m < mma_count(MODE, i)) md[f++] = mma_desc(MODE, i, m);
      }
#pragma unroll
      for (int f = 0; f < NM; ++f) {
        acc_first[f] = 0u;
#pragma unroll
        for (int e = 0; e < f; ++e)
          if (md[f].dgroup >= md[e].dgroup && md[f].dgroup < md[e].dgroup + 1 + md[e].wide)
            acc_first[f] = 1u;
      }
      const uint64_t a_desc = smem_desc_kmajor_sw128(sA);
      const uint64_t ring_desc = smem_desc_kmajor_noswizzle(sB, 0u, 128u);
      const uint32_t a_hi = (uint32_t)(a_desc >> 32), b_hi = (uint32_t)(ring_desc >> 32);
      // A descriptor step of one K-slice (block pair): two 8 KB blocks
      const uint32_t a_jp = 2 * (kBlockBytes >> 4);
      // chunk-invariant values, computed once: A descriptors, and the K-slices
      // per stage of full and last chunks (the issuer shares its scheduler with
      // busy warps, so integer work between stages sits on the MMA critical path)
      uint32_t a_lo[NM];
#pragma unroll
      for (int f = 0; f < NM; ++f)
        a_lo[f] = (uint32_t)a_desc + (uint32_t)(md[f].blk * (kBlockBytes >> 4) + md[f].pair * 2);
      const int ks_full = chunk_ks(F_in, F_out, 0), ks_last = chunk_ks(F_in, F_out, nchunks - 1);
      const int ns_full = nstage / ks_full, ns_last = nstage / ks_last;
      const int co_last = chunk_fields(F_out, nchunks - 1);
      uint32_t k = 0, ph = 0;
      bool ok = true;
      int ti = 0, c = 0;   // tile iteration and chunk of g
      for (int g = 0; g < total_chunks && ok; ++g) {
        const bool last_c = c == nchunks - 1;
        const int co = last_c ? co_last : kCoMax;
        const uint32_t buf = (uint32_t)g & 1u;
        // this chunk's descriptors first, then the wait for its accumulator
        const uint32_t id_n = H ? idesc_f16_f32(128, co) : idesc_bf16_f32(128, co);
        const uint32_t id_w = H ? idesc_f16_f32(128, 2 * co) : idesc_bf16_f32(128, 2 * co);
        const uint32_t half = (uint32_t)(co / 2);
        uint32_t dm[NM], b_lo[NM];
#pragma unroll
        for (int f = 0; f < NM; ++f) {
          dm[f] = buf * kAccBufCols + (uint32_t)md[f].dgroup * half;
          b_lo[f] = (uint32_t)ring_desc +
                    (uint32_t)((panel_offset(MODE, md[f].panel, co) + md[f].roff * (int)half * 16) >> 4) +
                    ((uint32_t)panel_rows(MODE, md[f].panel, co) << 16);   // LBO: one K-chunk of rows
        }
        const int ks = last_c ? ks_last : ks_full;
        const int ns = last_c ? ns_last : ns_full;
        const uint32_t slice = (uint32_t)(stage_bytes(MODE, co) >> 4);
        if (!mbar_wait_bounded_warp(bar_acc_empty(buf), (((uint32_t)g >> 1) & 1u) ^ 1u, fault,
                                    FAULT_WAIT_ACC_EMPTY, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
#pragma unroll
        for (int f = 0; f < NM; ++f) dm[f] += tmem_base;
        // ring stage s holds K-slices (block pairs) s*ks .. s*ks+ks-1, each
        // `slice` 16-byte units after the previous one; a_st is the A offset
        // of the stage's first K-slice
        uint32_t a_st = 0;
        for (int s = 0; s < ns && ok; ++s) {
          // a tile's first chunk also waits for the stage's block pairs of A
          for (int q = 0; q < ks && c == 0; ++q)
            if (!mbar_wait_bounded_warp(bar_a_full(s * ks + q), (uint32_t)ti & 1u, fault,
                                        FAULT_WAIT_A_FULL, kWaitLimitNs)) {
              ok = false;
              break;
            }
          if (!ok) break;
          // the weights have usually landed already: a non-blocking test
          // first, the bounded blocking wait only when they have not
          if (!__all_sync(0xffffffffu, mbar_test_wait(bar_b_full(k), ph)) &&
              !mbar_wait_bounded_warp(bar_b_full(k), ph, fault, FAULT_WAIT_B_FULL, kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t kb = k * ((uint32_t)slot_bytes >> 4);
          if (elect_one_sync()) {
            for (int q = 0; q < ks; ++q) {
              const uint32_t acc = s * ks + q > 0 ? 1u : 0u;
              const uint32_t qa = a_st + (uint32_t)q * a_jp, qb = kb + (uint32_t)q * slice;
#pragma unroll
              for (int f = 0; f < NM; ++f)
                mma_bf16_pair_w(dm[f], a_lo[f] + qa, a_hi, b_lo[f] + qb, b_hi,
                                (md[f].wide ? id_w : id_n) | (md[f].neg ? (1u << 14) : 0u),
                                acc | acc_first[f]);
            }
            mma_commit_pair_mc(bar_b_empty(k), 0x3);
          }
          __syncwarp();
          a_st += (uint32_t)ks * a_jp;
          if (++k == (uint32_t)nslots) {
            k = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one_sync()) mma_commit_pair_mc(bar_acc_full(buf), 0x3);
        __syncwarp();
        if (++c == nchunks) {
          c = 0;
          ++ti;
        }
      }
    }
  } else if (warp >= kDftWarp0 && warp < kDftWarp0 + kNumDftWarps) {
    // ------------------------------------------------------------ forward transform
    // Group grp (2 warps, 64 token rows) owns the block pairs jp with
    // pair_group(jp) = grp that the epilogue warps do not take: as each lands
    // (x_full), all 64 threads transform it in place and the group reports it
    // to the issuer (a_full on the leader CTA).
    const int grp = (warp - kDftWarp0) / kDftWarpsPerGroup;
    const int t = ((warp - kDftWarp0) % kDftWarpsPerGroup) * 32 + lane;  // token row in this CTA
    const uint32_t leader_a_full0 = mapa_shared(bar_a_full(0), 0);
    auto transform_tile = [&](int ti) -> bool {
      for (int jp = grp; jp < nstage; ++jp) {
        if (pair_by_epilogue<MODE>(jp) || pair_group<MODE>(jp) != grp) continue;
        if (!mbar_wait_bounded(bar_x_full(jp), (uint32_t)ti & 1u, fault, FAULT_WAIT_X_FULL,
                               kWaitLimitNs, kSleepNs))
          return false;
        uint8_t *r0 = gbase + (size_t)(2 * jp) * kBlockBytes + t * 128;
        transform_rows<MODE, H>(r0, r0 + kBlockBytes, t & 7, args.gelu);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) arrive_a_full(leader_a_full0 + 8u * (uint32_t)jp);
      }
      return true;
    };
    if constexpr (transform_warps_help_epilogue<MODE>()) {
      // transform warps 0..kD8HelpWarps-1 also take the odd 8-column groups of
      // every chunk's epilogue; the next tile's block pairs are transformed
      // before the share of a tile's last chunk (whose buffer the next tile's
      // first chunk does not use)
      const int wt = warp - kDftWarp0;
      const bool helper = wt < kD8HelpWarps;
      const int q4 = warp & 3;
      const int h = q4 >> 1;
      const int sub = wt >> 2;
      const int tq = lane & 3, tr = lane >> 2;
      const uint32_t leader_acc_empty0 = mapa_shared(bar_acc_empty(0), 0);
      uint8_t *const ybase = static_cast<uint8_t *>(args.y);
      bool ok = ntile_local == 0 || transform_tile(0);
      for (int g = 0; g < total_chunks && ok; ++g) {
        const int ti = g / nchunks, c = g % nchunks;
        if (c == nchunks - 1 && ti + 1 < ntile_local && !transform_tile(ti + 1)) {
          ok = false;
          break;
        }
        if (!helper) continue;
        const uint32_t buf = (uint32_t)g & 1u;
        if (!mbar_wait_bounded(bar_acc_full(buf), ((uint32_t)g >> 1) & 1u, fault,
                               FAULT_WAIT_ACC_FULL, kWaitLimitNs, kSleepNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
        const int half = chunk_fields(F_out, c) >> 1;
        const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32 + sub * 16) << 16) + buf * kAccBufCols;
        const int64_t tok0 = (int64_t)(pair + ti * npairs) * kTileTokens + (int64_t)rank * kRowsPerCta +
                             (q4 & 1) * 32 + sub * 16 + tr;
        const int field_base = c * kCoMax + h * half + 2 * tq;
        for (int fg = 8; fg < half; fg += 16) {
          if constexpr (MODE == kModeD8)
            d8_epilogue_group<H>(tb, fg, half, tok0, field_base, args.T, F_out, ybase, args.gelu);
          else
            neg16_epilogue_group(tb, fg, half, tok0, field_base, args.T, F_out, ybase, args.y_even);
        }
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(leader_acc_empty0 + 8u * buf);
      }
    } else {
      bool ok = true;
      for (int ti = 0; ti < ntile_local && ok; ++ti) {
        for (int jp = grp; jp < nstage; ++jp) {
          if (pair_by_epilogue<MODE>(jp) || pair_group<MODE>(jp) != grp) continue;
          if (!mbar_wait_bounded(bar_x_full(jp), (uint32_t)ti & 1u, fault, FAULT_WAIT_X_FULL,
                                 kWaitLimitNs, kSleepNs)) {
            ok = false;
            break;
          }
          uint8_t *r0 = gbase + (size_t)(2 * jp) * kBlockBytes + t * 128;
          transform_rows<MODE, H>(r0, r0 + kBlockBytes, t & 7, args.gelu);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) arrive_a_full(leader_a_full0 + 8u * (uint32_t)jp);
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // TMEM lane quarter q4 = warp % 4 holds token rows 32*(q4%2).. of this CTA
    // for the first (q4 < 2) or second half of each chunk's fields.  The two
    // warps of a quarter take 16 rows each.  A 16x256b load of coordinate
    // group kk gives thread t the columns 2(t%4), 2(t%4)+1 of rows t/4 and
    // t/4+8, i.e. 2 fields x 2 tokens; after 8 such loads each thread holds
    // all 8 coordinates of 4 (token, field) items, inverse-transforms them and
    // writes two 32-byte pieces of y (a quad covers a token's 8 fields, 128
    // contiguous bytes).
    const int q4 = warp & 3;
    const int h = q4 >> 1;
    const int sub = (warp - kEpiWarp0) >> 2;            // which 16 of the quarter's 32 rows
    const int tq = lane & 3, tr = lane >> 2;
    const uint32_t leader_acc_empty0 = mapa_shared(bar_acc_empty(0), 0);
    uint8_t *const ybase = static_cast<uint8_t *>(args.y);
    const int64_t T = args.T;
    // the block pairs this warp's help group transforms for tile iteration ti
    const int hgrp = (warp - kEpiWarp0) / kDftWarpsPerGroup;
    const int ht = ((warp - kEpiWarp0) % kDftWarpsPerGroup) * 32 + lane;
    const uint32_t leader_a_full0 = mapa_shared(bar_a_full(0), 0);
    auto help_transform = [&](int ti) -> bool {
      for (int jp = kDftGroups + hgrp; jp < nstage && pair_by_epilogue<MODE>(jp); jp += kEpiHelpGroups)
        if (!transform_pair_call<MODE, H>(gbase + (size_t)(2 * jp) * kBlockBytes, bar_x_full(jp),
                                          (uint32_t)ti & 1u, fault, ht, args.gelu,
                                          leader_a_full0 + 8u * (uint32_t)jp))
          return false;
      return true;
    };
    bool ok = true;
    for (int g = 0; g < total_chunks && ok; ++g) {
      // the first tile's helped block pairs before anything else; then, before
      // a tile's last chunk, whose epilogue the next tile's first chunk does
      // not wait for, the next tile's (with one chunk per tile, both at g = 0)
      if constexpr (epilogue_helps<MODE>()) {
        const bool last_c = g % nchunks == nchunks - 1;
        const int h0 = g == 0 ? 0 : (last_c ? g / nchunks + 1 : ntile_local);
        const int h1 = last_c ? g / nchunks + 1 : 0;
        for (int hti = h0; hti <= h1 && hti < ntile_local && ok; ++hti) ok = help_transform(hti);
        if (!ok) break;
      }
      const int tile = pair + (g / nchunks) * npairs;
      const int c = g % nchunks;
      const uint32_t buf = (uint32_t)g & 1u;
      if constexpr (MODE == kModeNegacyclic8) {
        // the even half's outputs that this warp reads in the next chunk's
        // epilogue (its 16 token rows, `half` fields each: one contiguous run
        // per row) are pulled into L2 a chunk ahead (the first chunk's at
        // once), so its loads there do not wait on DRAM
        for (int g1 = g == 0 ? 0 : g + 1; g1 <= g + 1 && g1 < total_chunks; ++g1) {
          const int c1 = g1 % nchunks;
          const int half1 = chunk_fields(F_out, c1) >> 1;
          const int64_t tok1 = (int64_t)(pair + (g1 / nchunks) * npairs) * kTileTokens +
                               (int64_t)rank * kRowsPerCta + (q4 & 1) * 32 + sub * 16 + lane;
          if (lane < 16 && tok1 < T)
            bulk_prefetch_l2(static_cast<const uint8_t *>(args.y_even) +
                                 ((size_t)tok1 * F_out + c1 * kCoMax + h * half1) * 16,
                             (uint32_t)half1 * 16u);
        }
      }
      if (!mbar_wait_bounded(bar_acc_full(buf), ((uint32_t)g >> 1) & 1u, fault,
                             FAULT_WAIT_ACC_FULL, kWaitLimitNs, kSleepNs)) {
        ok = false;
        break;
      }
      tcgen05_fence_after();
      const int co = chunk_fields(F_out, c);
      const int half = co >> 1;
      const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32 + sub * 16) << 16) + buf * kAccBufCols;
      const int64_t tok0 = (int64_t)tile * kTileTokens + (int64_t)rank * kRowsPerCta +
                           (q4 & 1) * 32 + sub * 16 + tr;
      const int field_base = c * kCoMax + h * half + 2 * tq;
      // D8: the epilogue warps take the even 8-column groups, transform warps
      // 0..7 the odd ones (kD8HelpWarps)
      for (int fg = 0; fg < half; fg += (transform_warps_help_epilogue<MODE>() ? 16 : 8)) {
        if constexpr (MODE == kModeD8) {
          d8_epilogue_group<H>(tb, fg, half, tok0, field_base, T, F_out, ybase, args.gelu);
          continue;
        }
        if constexpr (MODE == kModeNegacyclic8) {
          neg16_epilogue_group(tb, fg, half, tok0, field_base, T, F_out, ybase, args.y_even);
          continue;
        }
        if constexpr (MODE == kModeCyclic4) {
          // four coordinate groups; a thread's two columns are the two C_4
          // fields of one output super-field, for token rows tr and tr + 8
          uint32_t v4[4][4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tmem_ld_16x256b(tb + (uint32_t)(kk * half + fg), v4[kk]);
          tmem_wait_ld();
          float2 z[8], yv[8];   // lane x: token row tr, lane y: tr + 8
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int q = group_coord(MODE, kk);
            z[q] = make_float2(__uint_as_float(v4[kk][0]), __uint_as_float(v4[kk][2]));       // field 2tq
            z[4 + q] = make_float2(__uint_as_float(v4[kk][1]), __uint_as_float(v4[kk][3]));   // field 2tq + 1
          }
          inv_cyclic4x2(z, yv);
          uint32_t wa[4], wb[4];
#pragma unroll
          for (int p2 = 0; p2 < 4; ++p2) {
            wa[p2] = pack_x2<H>(yv[2 * p2].x, yv[2 * p2 + 1].x);
            wb[p2] = pack_x2<H>(yv[2 * p2].y, yv[2 * p2 + 1].y);
          }
          // the super-field's 8 outputs (two C_4 fields x 4 slots) are 16 contiguous bytes
#pragma unroll
          for (int r8 = 0; r8 < 2; ++r8) {
            const int64_t tok = tok0 + 8 * r8;
            if (tok < T) {
              uint8_t *dst = ybase + (tok * F_out + field_base + fg) * 8;
              *reinterpret_cast<uint4 *>(dst) =
                  r8 ? make_uint4(wb[0], wb[1], wb[2], wb[3]) : make_uint4(wa[0], wa[1], wa[2], wa[3]);
            }
          }
        } else {
          uint32_t v[8][4];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) tmem_ld_16x256b(tb + (uint32_t)(kk * half + fg), v[kk]);
          tmem_wait_ld();
          uint32_t w[4][4];
#pragma unroll
          for (int ip = 0; ip < 4; ip += 2) {     // items ip, ip + 1 as the two float2 lanes
            float2 z[8], yv[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              z[group_coord(MODE, kk)] =
                  make_float2(__uint_as_float(v[kk][ip]), __uint_as_float(v[kk][ip + 1]));
            if (MODE == kModeCyclic8)
              inv_cyclic8(z, yv);
            else if ((args.gelu & (kD8OutFourier | kD8Gelu)) == kD8OutFourier) {
#pragma unroll
              for (int gg = 0; gg < 8; ++gg) yv[gg] = z[gg];   // coordinates out as they are
            } else {
              inv_d8(z, yv);
              if (args.gelu & kD8Gelu) {
#pragma unroll
                for (int gg = 0; gg < 8; ++gg) yv[gg] = gelu_tanh2(yv[gg]);
              }
              if (args.gelu & kD8OutFourier) {   // the GELU round trip: back to coordinates
                float2 zz[8];
                fwd_d8(yv, zz);
#pragma unroll
                for (int gg = 0; gg < 8; ++gg) yv[gg] = zz[gg];
              }
            }
            if (args.gelu & kOutF32) {
              // fp32 y: item ip (lane x) and ip + 1 (lane y) are 32 contiguous bytes each;
              // items 0, 1: token tok0, fields f, f + 1; items 2, 3: token tok0 + 8
              const int64_t tok = tok0 + 8 * (ip >> 1);
              if (tok < T) {
                uint32_t a[4], b[4], c2[4], d[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  a[q] = __float_as_uint(yv[q].x);
                  b[q] = __float_as_uint(yv[4 + q].x);
                  c2[q] = __float_as_uint(yv[q].y);
                  d[q] = __float_as_uint(yv[4 + q].y);
                }
                uint8_t *dst = ybase + (tok * F_out + field_base + fg) * 32;
                st_global_v8(dst, a, b);
                st_global_v8(dst + 32, c2, d);
              }
              continue;
            }
#pragma unroll
            for (int p2 = 0; p2 < 4; ++p2) {
              w[ip][p2] = pack_x2<H>(yv[2 * p2].x, yv[2 * p2 + 1].x);
              w[ip + 1][p2] = pack_x2<H>(yv[2 * p2].y, yv[2 * p2 + 1].y);
            }
          }
          if (args.gelu & (kOutF32 | kCombine16)) continue;   // stored above (kCombine16: never here)
          // items 0, 1: token tok0, fields f, f+1; items 2, 3: token tok0 + 8
#pragma unroll
          for (int r8 = 0; r8 < 2; ++r8) {
            const int64_t tok = tok0 + 8 * r8;
            if (tok < T) {
              uint8_t *dst = ybase + (tok * F_out + field_base + fg) * 16;
              st_global_v8(dst, w[2 * r8], w[2 * r8 + 1]);
            }
          }
        }
      }
      // the columns are in registers (tcgen05.wait::ld): a relaxed arrive
      // frees them without waiting for this warp's y stores to be performed
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(leader_acc_empty0 + 8u * buf);
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  if (fault_raised(fault)) {
    // a bounded wait of this launch gave up: give copies still in flight time to land
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kWarpProd) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- packing

// (weight sources, D8 blocks and the spectral block values: tc_pack_math.cuh)

// One CUDA block per (stage jp, CTA half) of chunk c; the thread loop walks
// the stage's bf16 elements in shared-memory image order.
// WT: the weight's type (0 bf16, 1 fp16, 2 fp32); H: the stored operand type
// (bf16 or fp16).  split_cin > 0 (cyclic mode, fp32 weights): the layer's
// input fields are three blocks of split_cin, [hi | hi | lo] of the spectrum,
// hi = bf16(v), lo = bf16(v - hi), against activations [X_hi | X_lo | X_hi].
template <int MODE, bool H, int WT = (H ? 1 : 0)>
__global__ void pack_b_kernel(const void *__restrict__ Wc, D8Blocks d8, int F_in,
                              int F_out, int wsrc, int c, uint16_t *__restrict__ dst, int split_cin = 0,
                              int split_off = 0, int split_full = 0) {
  const int co = chunk_fields(F_out, c);
  const int hc = co / 2;
  const int jp = blockIdx.x >> 1, hh = blockIdx.x & 1;
  const int64_t off = stage_offset(MODE, F_in, F_out, c, jp, hh);  // bytes
  const int nel = stage_bytes(MODE, co) / 2;
  for (int e = threadIdx.x; e < nel; e += blockDim.x) {
    int k = 0;
    while (k + 1 < num_panels(MODE) && 2 * e >= panel_offset(MODE, k + 1, co)) ++k;
    const int w = e - panel_offset(MODE, k, co) / 2;  // element within panel k
    double val;
    int split_blk = 0;   // with split_cin: which of the three input-field blocks
    if (MODE == kModeCyclic4) {
      // row r = k / 3 of the block pair (its 16 C_4 fields 32jp + 16r ..); a
      // K-chunk kc holds the even (kc = 0) or odd fields, element el = field 2el + kc
      const int r = k / 3, kind = k % 3;
      if (kind < 2) {   // W0 or W2: [K-chunk 2][hc rows][8]
        const int kc = w / (hc * 8), row = (w / 8) % hc, el = w % 8;
        const int o = c * kCoMax + hh * hc + row;
        const int i = 32 * jp + 16 * r + 2 * el + kc;
        const int cc = kind == 0 ? 0 : 3;
        val = c4_block_value<WT>(Wc, 2 * F_in, F_out, wsrc, cc, o, cc, i);
      } else {          // bin 1: [K-chunk 2][co rows: Wi (row < hc), Wr][8]
        const int kc = w / (co * 8), row = (w / 8) % co, el = w % 8;
        const int o = c * kCoMax + hh * hc + (row % hc);
        const int i = 32 * jp + 16 * r + 2 * el + kc;
        val = row < hc ? c4_block_value<WT>(Wc, 2 * F_in, F_out, wsrc, 2, o, 1, i)
                       : c4_block_value<WT>(Wc, 2 * F_in, F_out, wsrc, 1, o, 1, i);
      }
    } else if (MODE == kModeNegacyclic8) {
      // bin b = k: [K-chunk 2][co rows: Wi (r < hc), Wr (r >= hc)][8]
      const int kc = w / (co * 8), r = (w / 8) % co, el = w % 8;
      const int o = c * kCoMax + hh * hc + (r % hc);
      const int i = (2 * jp + kc) * 8 + el;
      const int cre = 2 * k, cim = 2 * k + 1;
      val = r < hc ? block_value<MODE, WT>(Wc, d8, F_in, F_out, wsrc, cim, o, cre, i)
                   : block_value<MODE, WT>(Wc, d8, F_in, F_out, wsrc, cre, o, cre, i);
    } else if (MODE == kModeCyclic8 ? k < 2 : k < 4) {
      // [K-chunk 2][hc rows][8]: K-chunk kc = block 2jp + kc, row r -> output field
      const int kc = w / (hc * 8), r = (w / 8) % hc, el = w % 8;
      const int o = c * kCoMax + hh * hc + r;
      int i = (2 * jp + kc) * 8 + el, Fw = F_in;
      if (split_cin > 0) {   // input field split_off + i % split_cin of a split_full-wide W
        split_blk = i / split_cin;
        i = split_off + i % split_cin;
        Fw = split_full > 0 ? split_full : split_cin;
      }
      const int cr = MODE == kModeCyclic8 ? (k == 0 ? 0 : 7) : k;
      val = block_value<MODE, WT>(Wc, d8, Fw, F_out, wsrc, cr, o, cr, i);
    } else if (MODE == kModeCyclic8) {
      // complex bin b = k - 1: [K-chunk 2][co rows: Wi (r < hc), Wr (r >= hc)][8],
      // Wr = 2 Re W_b, Wi = 2 Im W_b (block_value's [[Wr, -Wi], [Wi, Wr]])
      const int kc = w / (co * 8), r = (w / 8) % co, el = w % 8;
      const int o = c * kCoMax + hh * hc + (r % hc);
      int i = (2 * jp + kc) * 8 + el, Fw = F_in;
      if (split_cin > 0) {   // input field split_off + i % split_cin of a split_full-wide W
        split_blk = i / split_cin;
        i = split_off + i % split_cin;
        Fw = split_full > 0 ? split_full : split_cin;
      }
      const int bin = k - 1;
      const int cre = 2 * bin - 1, cim = 2 * bin;
      val = r < hc ? block_value<MODE, WT>(Wc, d8, Fw, F_out, wsrc, cim, o, cre, i)
                   : block_value<MODE, WT>(Wc, d8, Fw, F_out, wsrc, cre, o, cre, i);
    } else {
      // D8 E, K-step ks = 2jp + (k - 4): [K-chunk = b][co rows = (b', field)][8 fields]
      const int ks = 2 * jp + (k - 4);
      const int kc = w / (co * 8), r = (w / 8) % co, el = w % 8;
      const int bo = r >= hc ? 1 : 0;
      const int o = c * kCoMax + hh * hc + (r % hc);
      const int i = ks * 8 + el;
      val = block_value<MODE, WT>(Wc, d8, F_in, F_out, wsrc, 4 + bo, o, 4 + kc, i);
    }
    if (split_cin > 0 && split_blk == 2)   // the lo part: what bf16 misses of the value
      val -= (double)__bfloat162float(__float2bfloat16_rn((float)val));
    dst[off / 2 + e] = H ? __half_as_ushort(__float2half_rn((float)val))
                         : __bfloat16_as_ushort(__float2bfloat16_rn((float)val));
  }
}

template <int MODE, bool H = false, int WT = (H ? 1 : 0)>
int launch_pack(const void *Wc, D8Blocks d8, int F_in, int F_out, int wsrc, void *dst,
                cudaStream_t s, int split_cin = 0, int split_off = 0, int split_full = 0) {
  for (int c = 0; c < num_chunks(F_out); ++c)
    pack_b_kernel<MODE, H, WT><<<(F_in / 16) * 2, 256, 0, s>>>(Wc, d8, F_in, F_out, wsrc, c,
                                                               static_cast<uint16_t *>(dst), split_cin,
                                                               split_off, split_full);
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

struct DevCache {   // per mode, per operand type (bf16, fp16)
  int max_clusters[4][2] = {};
  bool attr_set[4][2] = {};
};
std::mutex g_cache_mu;
DevCache g_cache[64];

template <int MODE, bool H = false>
int launch_tc(const void *x, const void *Bpack, void *y, int64_t T, int F_in, int F_out, int gelu, int x_ld,
              cudaStream_t s, const void *y_even = nullptr) {
  if (T >= (int64_t)0x7fffff00LL) return set_error(EQLIN_ERR_UNSUPPORTED, "T too large");
  if (((uintptr_t)y & 31u) != 0)
    return set_error(EQLIN_ERR_ALIGN, "tensor-core path needs y 32-byte aligned");
  const int ntiles = (int)((T + kTileTokens - 1) / kTileTokens);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(EQLIN_ERR_CUDA, "cudaGetDevice failed");
  auto kern = spectral8_tc_kernel<MODE, H>;
  const int smem_max = kSmemLimit;
  int maxc = 0;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    DevCache &dc = g_cache[dev];
    if (!dc.attr_set[MODE][H]) {
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
      dc.max_clusters[MODE][H] = n;
      dc.attr_set[MODE][H] = true;
    }
    maxc = dc.max_clusters[MODE][H];
  }
  CUtensorMap mx, mbf, mbl;
  // x rows are x_ld fields apart (F_in unless the layer reads a column slice)
  int rc = make_map_2d(&mx, x, (uint64_t)F_in * 8, (uint64_t)T, (uint64_t)x_ld * 16, 64,
                       kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  const int64_t bbytes = packed_bytes(MODE, F_in, F_out);
  const int full_rows = chunk_stage_bytes(MODE, F_in, F_out, 0) / kBRow;
  const int last_rows = chunk_stage_bytes(MODE, F_in, F_out, num_chunks(F_out) - 1) / kBRow;
  rc = make_map_2d(&mbf, Bpack, kBRow / 2, (uint64_t)(bbytes / kBRow), kBRow, kBRow / 2,
                   (uint32_t)full_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = make_map_2d(&mbl, Bpack, kBRow / 2, (uint64_t)(bbytes / kBRow), kBRow, kBRow / 2,
                   (uint32_t)last_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  const RingShape ring = ring_shape(MODE, F_in, F_out);
  if (ring.nslots < 2) return set_error(EQLIN_ERR_UNSUPPORTED, "weight ring does not fit");
  TcArgs a;
  a.y = y;
  a.nslots = ring.nslots;
  a.slot_bytes = ring.slot_bytes;
  a.T = T;
  a.F_in = F_in;
  a.F_out = F_out;
  a.ntiles = ntiles;
  a.gelu = gelu;
  a.y_even = y_even;
  a.epoch = next_launch_epoch();
  const int npairs = ntiles < maxc ? ntiles : maxc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * npairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes_for(F_in, ring);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mx, mbf, mbl, a);
  if (e != cudaSuccess)
    return set_error(EQLIN_ERR_CUDA, "tensor-core launch: %s", cudaGetErrorString(e));
  return check_launch("spectral8_tc_kernel");
}

// ---------------------------------------------------------------- C_16 in two passes
// A C_16 layer splits exactly into a C_8 cyclic layer on e_h = x_h + x_{h+8}
// and a C_8 negacyclic layer on d_h = x_h - x_{h+8} (X(z) mod z^16 - 1 =
// (z^8 - 1)(z^8 + 1)); with the 1/2 folded into both weight spectra,
// y_g = Y_e,g + Y_o,g and y_{g+8} = Y_e,g - Y_o,g.  Each half has the C_8
// kernel's A footprint, which the 16-slot layer's would not fit beside a
// weight ring.  The even half's output goes to the workspace; the odd half's
// epilogue reads it and writes the C_16 output (kCombine16).

// x [T][F][16] -> e, d [T][F][8] (bf16, fp32 arithmetic), one (token, field) per thread.
__global__ void c16_fold_kernel(const __nv_bfloat16 *__restrict__ x, __nv_bfloat16 *__restrict__ e,
                                __nv_bfloat16 *__restrict__ d, int64_t n) {
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
    const uint4 lo = reinterpret_cast<const uint4 *>(x)[2 * p];
    const uint4 hi = reinterpret_cast<const uint4 *>(x)[2 * p + 1];
    float2 a[8];
    unpack_bf16x8_pair(lo, hi, a);          // a[h] = (x_h, x_{h+8})
    uint32_t ew[4], dw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      ew[k] = pack_bf16x2(a[2 * k].x + a[2 * k].y, a[2 * k + 1].x + a[2 * k + 1].y);
      dw[k] = pack_bf16x2(a[2 * k].x - a[2 * k].y, a[2 * k + 1].x - a[2 * k + 1].y);
    }
    reinterpret_cast<uint4 *>(e)[p] = make_uint4(ew[0], ew[1], ew[2], ew[3]);
    reinterpret_cast<uint4 *>(d)[p] = make_uint4(dw[0], dw[1], dw[2], dw[3]);
  }
}

size_t c16_region(int64_t T, int F) { return ((size_t)T * F * 16 + 255) / 256 * 256; }

// fp32 C_8 on the bf16 MMAs works on slices of at most kF32Slice input fields:
// a slice of w fields becomes a 3w-wide layer, which must fit the resident A
// operand (kMaxFin fields).  Slice j holds input fields j kF32Slice ..
constexpr int kF32Slice = 48;
__host__ __device__ inline int f32_nslices(int Cin) { return (Cin + kF32Slice - 1) / kF32Slice; }
__host__ __device__ inline int f32_slice_w(int Cin, int j) {
  const int r = Cin - j * kF32Slice;
  return r < kF32Slice ? r : kF32Slice;
}
static_assert(3 * kF32Slice <= kMaxFin, "a split slice fits the A operand");
// Byte offset of slice j's packed weights (each slice's block 256-byte aligned).
size_t f32_pack_offset(int Cin, int Cout, int j) {
  size_t off = 0;
  for (int k = 0; k < j; ++k)
    off += ((size_t)packed_bytes(kModeCyclic8, 3 * f32_slice_w(Cin, k), Cout) + 255) / 256 * 256;
  return off;
}

// The fp32 spectrum X of each field is split as X_hi = bf16(X), X_lo =
// bf16(X - X_hi) and written, per slice of w input fields, as three blocks of
// w "fields" [X_hi | X_lo | X_hi] (slice j from field 3 j kF32Slice of a row
// of 3 Cin fields); against weights [W_hi | W_hi | W_lo] one pass of the MMAs
// over a slice sums X_hi W_hi + X_lo W_hi + X_hi W_lo.  One thread per (token,
// pair of fields), the pair as the float2 lanes (a pair never straddles a
// slice: slices and Cin are multiples of 16).
__global__ void c8_split_prepass_kernel(const float *__restrict__ x, __nv_bfloat16 *__restrict__ a,
                                        int64_t T, int Cin) {
  const int half = Cin / 2;
  const int64_t n = T * half;
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = p / half;
    const int i = 2 * (int)(p % half);
    const float4 *src = reinterpret_cast<const float4 *>(x + ((size_t)t * Cin + i) * 8);
    const float4 a0 = src[0], a1 = src[1], b0 = src[2], b1 = src[3];
    const float2 xv[8] = {make_float2(a0.x, b0.x), make_float2(a0.y, b0.y), make_float2(a0.z, b0.z),
                          make_float2(a0.w, b0.w), make_float2(a1.x, b1.x), make_float2(a1.y, b1.y),
                          make_float2(a1.z, b1.z), make_float2(a1.w, b1.w)};
    float2 z[8];
    fwd_cyclic8(xv, z);
    uint32_t hi0[4], hi1[4], lo0[4], lo1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 u = z[2 * k], v = z[2 * k + 1];
      const float ux = __bfloat162float(__float2bfloat16_rn(u.x)), vx = __bfloat162float(__float2bfloat16_rn(v.x));
      const float uy = __bfloat162float(__float2bfloat16_rn(u.y)), vy = __bfloat162float(__float2bfloat16_rn(v.y));
      hi0[k] = pack_bf16x2(ux, vx);
      hi1[k] = pack_bf16x2(uy, vy);
      lo0[k] = pack_bf16x2(u.x - ux, v.x - vx);
      lo1[k] = pack_bf16x2(u.y - uy, v.y - vy);
    }
    const int j = i / kF32Slice, li = i - j * kF32Slice, w = f32_slice_w(Cin, j);
    uint4 *row = reinterpret_cast<uint4 *>(a + (size_t)t * 3 * Cin * 8) + 3 * j * kF32Slice;
    const uint4 h0 = make_uint4(hi0[0], hi0[1], hi0[2], hi0[3]), h1 = make_uint4(hi1[0], hi1[1], hi1[2], hi1[3]);
    row[li] = h0;
    row[li + 1] = h1;
    row[w + li] = make_uint4(lo0[0], lo0[1], lo0[2], lo0[3]);
    row[w + li + 1] = make_uint4(lo1[0], lo1[1], lo1[2], lo1[3]);
    row[2 * w + li] = h0;
    row[2 * w + li + 1] = h1;
  }
}

// y += p over n4 float4s (the fp32 partial output of one more slice).
__global__ void f32_accumulate_kernel(float *__restrict__ y, const float *__restrict__ p, int64_t n4) {
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n4; k += (int64_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<float4 *>(y)[k];
    const float4 b = reinterpret_cast<const float4 *>(p)[k];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    reinterpret_cast<float4 *>(y)[k] = a;
  }
}

}  // namespace

// ---------------------------------------------------------------- bounded-wait self-test

// One warp waits, with the same bounded wait every kernel here uses, on an
// mbarrier of arrival count 1.  arrive = 1: thread 0 arrives first, so the
// phase completes and the wait returns at once.  arrive = 0: nothing ever
// arrives; the wait gives up after limit_ns and records FAULT_SELFTEST.
// *elapsed_ns receives the wait's duration (globaltimer).
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int arrive, unsigned int epoch,
                                             unsigned long long *elapsed_ns) {
  using namespace tc;
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) mbar_init(bar, 1);
  __syncthreads();   // the barrier is CTA-local: the block barrier publishes its init
  if (arrive && threadIdx.x == 0)
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
  __syncwarp();
  const uint64_t t0 = globaltimer_ns();
  const FaultCtx fault{g_fault_state, epoch};
  mbar_wait_bounded_warp(bar, 0u, fault, (unsigned int)FAULT_SELFTEST, limit_ns);
  const uint64_t t1 = globaltimer_ns();
  if (threadIdx.x == 0 && elapsed_ns) *elapsed_ns = (unsigned long long)(t1 - t0);
}

int launch_bounded_wait_selftest(uint64_t limit_ns, int arrive, unsigned long long *elapsed_ns,
                                 cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns, arrive, next_launch_epoch(), elapsed_ns);
  return check_launch("bounded-wait self-test");
}

// ---------------------------------------------------------------- interface

int tma_map_2d_bf16(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  return make_map_2d(m, ptr, inner, outer, row_bytes, box_inner, box_outer,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

int fault_word_address(unsigned int **out) {
  static std::mutex mu;
  static unsigned int *addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(EQLIN_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fault_state);
    if (e != cudaSuccess || !p)
      return set_error(EQLIN_ERR_CUDA, "cudaGetSymbolAddress of the fault word: %s",
                       cudaGetErrorString(e));
    addr[dev] = static_cast<unsigned int *>(p);
  }
  *out = addr[dev];
  return EQLIN_OK;
}

bool cyclic_tc_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && N == 8 && tc_shape_ok(Cin, Cout);
}

// p4 on the fused kernel: bf16, Cin C_4 fields in 32..320 (a multiple of 32,
// i.e. whole block pairs of super-fields), Cout a multiple of 32.
bool cyclic4_tc_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && N == 4 && Cin % 32 == 0 && tc_shape_ok(Cin / 2, Cout);
}

size_t cyclic4_tc_bytes(int Cin, int Cout) { return (size_t)packed_bytes(kModeCyclic4, Cin / 2, Cout); }

int launch_cyclic4_tc_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s) {
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  return launch_pack<kModeCyclic4>(W, none, Cin / 2, Cout, adjoint, dst, s);
}

int launch_cyclic4_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout, cudaStream_t s) {
  return launch_tc<kModeCyclic4>(x, Bpack, y, T, Cin / 2, Cout, 0, Cin / 2, s);
}

// fp32 C_8 through the split, slice by slice: slice 0 writes y, every later
// slice its fp32 partial output, which is added to y (a fixed order, so the
// result is deterministic).
bool cyclic_tc_f32_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_F32 && N == 8 && Cin >= 16 && Cin % 16 == 0 &&
         tc_shape_ok(3 * f32_slice_w(Cin, 0), Cout);
}

size_t cyclic_tc_f32_bytes(int Cin, int Cout) { return f32_pack_offset(Cin, Cout, f32_nslices(Cin)); }

size_t cyclic_tc_f32_workspace_bytes(int64_t T, int Cin, int Cout) {
  return c16_region(T, 3 * Cin) + (f32_nslices(Cin) > 1 ? ((size_t)T * Cout * 32 + 255) / 256 * 256 : 0);
}

int launch_cyclic_tc_f32_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s) {
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  for (int j = 0; j < f32_nslices(Cin); ++j) {
    const int w = f32_slice_w(Cin, j);
    const int rc = launch_pack<kModeCyclic8, false, 2>(W, none, 3 * w, Cout, adjoint,
                                                       static_cast<char *>(dst) + f32_pack_offset(Cin, Cout, j),
                                                       s, w, j * kF32Slice, Cin);
    if (rc != EQLIN_OK) return rc;
  }
  return EQLIN_OK;
}

int launch_cyclic_tc_f32(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                         void *workspace, cudaStream_t s) {
  const int64_t n = T * (Cin / 2);
  const unsigned g = (unsigned)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  c8_split_prepass_kernel<<<g, 256, 0, s>>>(static_cast<const float *>(x),
                                            static_cast<__nv_bfloat16 *>(workspace), T, Cin);
  int rc = check_launch("fp32 split pre-pass");
  if (rc != EQLIN_OK) return rc;
  float *part = reinterpret_cast<float *>(static_cast<char *>(workspace) + c16_region(T, 3 * Cin));
  const int64_t n4 = T * (int64_t)Cout * 2;
  const unsigned ga = (unsigned)((n4 + 255) / 256 < 148 * 16 ? (n4 + 255) / 256 : 148 * 16);
  for (int j = 0; j < f32_nslices(Cin); ++j) {
    const int w = f32_slice_w(Cin, j);
    const char *aj = static_cast<const char *>(workspace) + (size_t)3 * j * kF32Slice * 16;
    const char *bj = static_cast<const char *>(Bpack) + f32_pack_offset(Cin, Cout, j);
    rc = launch_tc<kModeCyclic8>(aj, bj, j == 0 ? y : part, T, 3 * w, Cout, kInFourier | kOutF32, 3 * Cin, s);
    if (rc != EQLIN_OK) return rc;
    if (j == 0) continue;
    f32_accumulate_kernel<<<ga, 256, 0, s>>>(static_cast<float *>(y), part, n4);
    rc = check_launch("fp32 slice accumulation");
    if (rc != EQLIN_OK) return rc;
  }
  return EQLIN_OK;
}

bool cyclic_tc_f16_supported(int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_F16 && N == 8 && tc_shape_ok(Cin, Cout);
}

bool d8_tc_supported(int C, int dtype) {
  return dtype == EQLIN_BF16 && C % 8 == 0 && tc_shape_ok(C / 8, C / 8);
}

size_t cyclic_tc_bytes(int, int Cin, int Cout) {
  return (size_t)packed_bytes(kModeCyclic8, Cin, Cout);
}

size_t d8_tc_bytes(int C) { return (size_t)packed_bytes(kModeD8, C / 8, C / 8); }

bool cyclic16_tc_supported(int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && tc_shape_ok(Cin, Cout);
}

size_t cyclic16_tc_bytes(int Cin, int Cout) {
  return 2 * (size_t)packed_bytes(kModeCyclic8, Cin, Cout);
}

size_t cyclic16_tc_workspace_bytes(int64_t T, int Cin, int Cout) {
  return 2 * c16_region(T, Cin) + c16_region(T, Cout);   // e, d, ye
}

int launch_cyclic16_tc_pack(const void *W, int Cin, int Cout, int adjoint, void *dst, cudaStream_t s) {
  static_assert(kModeCyclic8 != kModeNegacyclic8, "two modes");
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  const auto *Wc = static_cast<const __nv_bfloat16 *>(W);
  int rc = launch_pack<kModeCyclic8>(Wc, none, Cin, Cout, adjoint ? kWsrcFoldEvenAdj : kWsrcFoldEven, dst, s);
  if (rc != EQLIN_OK) return rc;
  return launch_pack<kModeNegacyclic8>(Wc, none, Cin, Cout, adjoint ? kWsrcFoldOddAdj : kWsrcFoldOdd,
                                       static_cast<char *>(dst) + packed_bytes(kModeCyclic8, Cin, Cout), s);
}

int launch_cyclic16_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout,
                       void *workspace, cudaStream_t s) {
  char *ws = static_cast<char *>(workspace);
  auto *e = reinterpret_cast<__nv_bfloat16 *>(ws);
  auto *d = reinterpret_cast<__nv_bfloat16 *>(ws + c16_region(T, Cin));
  auto *ye = reinterpret_cast<__nv_bfloat16 *>(ws + 2 * c16_region(T, Cin));
  const int64_t nin = T * Cin;
  const unsigned gi = (unsigned)((nin + 255) / 256 < 148 * 16 ? (nin + 255) / 256 : 148 * 16);
  c16_fold_kernel<<<gi, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), e, d, nin);
  int rc = check_launch("C_16 fold");
  if (rc != EQLIN_OK) return rc;
  rc = launch_tc<kModeCyclic8>(e, Bpack, ye, T, Cin, Cout, 0, Cin, s);
  if (rc != EQLIN_OK) return rc;
  return launch_tc<kModeNegacyclic8>(d, static_cast<const char *>(Bpack) + packed_bytes(kModeCyclic8, Cin, Cout),
                                     y, T, Cin, Cout, kCombine16, Cin, s, ye);
}

int launch_cyclic_tc_pack(const void *W, int, int Cin, int Cout, int adjoint, int dtype, void *dst,
                          cudaStream_t s) {
  D8Blocks none = {{nullptr, nullptr, nullptr, nullptr, nullptr}};
  if (dtype == EQLIN_F16) return launch_pack<kModeCyclic8, true>(W, none, Cin, Cout, adjoint, dst, s);
  return launch_pack<kModeCyclic8>(W, none, Cin, Cout, adjoint, dst, s);
}

int launch_d8_tc_pack(const void *const w[5], int C, void *dst, cudaStream_t s) {
  D8Blocks d8;
  for (int k = 0; k < 5; ++k) d8.w[k] = static_cast<const __nv_bfloat16 *>(w[k]);
  d8.ld1 = C / 8;
  d8.ldE = 2 * (C / 8);
  return launch_pack<kModeD8>(nullptr, d8, C / 8, C / 8, 0, dst, s);
}

int launch_cyclic_tc(const void *x, const void *Bpack, void *y, int64_t T, int Cin, int Cout, int dtype,
                     cudaStream_t s) {
  if (dtype == EQLIN_F16) return launch_tc<kModeCyclic8, true>(x, Bpack, y, T, Cin, Cout, 0, Cin, s);
  return launch_tc<kModeCyclic8>(x, Bpack, y, T, Cin, Cout, 0, Cin, s);
}

int launch_d8_tc(const void *x, const void *Bpack, void *y, int64_t T, int C, int gelu,
                 cudaStream_t s) {
  return launch_tc<kModeD8>(x, Bpack, y, T, C / 8, C / 8, gelu, C / 8, s);
}

bool d8_fourier_tc_supported(int F_in, int F_out, int dtype) {
  return dtype == EQLIN_BF16 && tc_shape_ok(F_in, F_out);
}

size_t d8_fourier_tc_bytes(int F_in, int F_out) { return (size_t)packed_bytes(kModeD8, F_in, F_out); }

// Column slice [k0, k0 + F_slice) of a Fourier-domain layer's blocks (all
// F_total input fields wide), packed as a layer of F_slice input fields.
int launch_d8_fourier_tc_pack(const void *const w[5], int F_total, int k0, int F_slice, int F_out,
                              void *dst, cudaStream_t s) {
  D8Blocks d8;
  for (int k = 0; k < 4; ++k) d8.w[k] = static_cast<const __nv_bfloat16 *>(w[k]) + k0;
  d8.w[4] = static_cast<const __nv_bfloat16 *>(w[4]) + 2 * k0;
  d8.ld1 = F_total;
  d8.ldE = 2 * F_total;
  return launch_pack<kModeD8>(nullptr, d8, F_slice, F_out, 0, dst, s);
}

// z rows are z_ld fields apart: a column slice of wider features reads its
// F_in fields at z + 8 k0 with z_ld = the full width.
int launch_d8_fourier_tc(const void *z, const void *Bpack, void *y, int64_t T, int F_in, int F_out,
                         int roundtrip_gelu, int z_ld, cudaStream_t s) {
  return launch_tc<kModeD8>(z, Bpack, y, T, F_in, F_out,
                            kD8InFourier | kD8OutFourier | (roundtrip_gelu ? kD8Gelu : 0), z_ld, s);
}

}  // namespace eqlin
