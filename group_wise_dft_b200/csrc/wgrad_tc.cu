// Weight gradient of the cyclic C_8 layer on tcgen05 tensor cores.
//
// For y[t,o,g] = sum_i sum_h W[o,i,(g-h) mod 8] x[t,i,h] the gradient of
// sum(dy * y) with respect to W is a token sum of circular cross-correlations,
// which the cross-correlation theorem turns into one product per frequency bin
// (the backward counterpart of Flash EQ-Linear, Methodology > Algorithmic
// Approach):
//     C_k[o,i] = sum_t DY_k[t,o] conj(X_k[t,i]),   k = 0..4,
// with X_k, DY_k the half spectra of each field.  Per real coordinate c of the
// half spectrum ([Re 0, Re 1, Im 1, Re 2, Im 2, Re 3, Im 3, Re 4]) that is a
// GEMM over tokens:
//     real bins:    C_c  = sum_t DY_c X_c
//     complex bins: Re C = sum_t (DYr Xr + DYi Xi),  Im C = sum_t (DYi Xr - DYr Xi).
// This kernel computes the C_c, split over token ranges, into the fp32 partial
// workspace [S][Cout][Cin][8] that the CUDA-core path also fills; the same
// fixed-order reduction and inverse transform (simt_wgrad.cu) finish dW.
//
// Work unit: (token split s, tile of 128 output fields x 128 input fields).
// CTA pair (cluster of 2, tcgen05 cta_group::2, M = 128): CTA r holds output
// fields 64r..64r+63 of the tile as the MMA's M rows; the input fields are two
// subtiles of 64, CTA r holding fields 32r..32r+31 of each as its B rows (its
// x boxes 0..7, one box apart), so one MMA of N = 128 covers both subtiles
// (N = 64 when the tile's second subtile holds no field).  TMEM: coordinate c
// at columns 64 c; lanes 0..63 hold the products with CTA 0's B rows, lanes
// 64..127 those with CTA 1's (column 32 st + j: subtile st, field j of the
// CTA's 32).  512 columns; the accumulators stay resident for the whole split.
// One N = 128 MMA reads A once for both subtiles: 32.5 cycles against 2 x 25.5
// for two N = 64 MMAs (the MMAs are bound by their shared-memory operand reads).
//
// Pipeline per CTA, kWtStages slots of kWtTk = 32 tokens:
//   producer warp   TMA-loads the slot's dy (8 boxes of 8 output fields) and
//                   x (8 boxes of 8 input fields), each box kWtTk tokens x
//                   128 bytes with the 128-byte swizzle
//   18 transform    in place: each 1 KB atom (8 tokens x 8 fields) is read
//   warps           whole, transformed (fwd_cyclic8, two tokens per thread as
//                   the float2 lanes), and rewritten as 8 core matrices, one
//                   per coordinate c (atom + 128 c: 8 field rows x 8 tokens),
//                   so coordinate c of the whole slot is a K-major operand with
//                   K-chunk stride 1 KB and 8-row-group stride one box
//   1 MMA issuer    (leader CTA) 14 MMAs of N = 128 per 16 tokens; in the
//                   peer CTA the same warp forwards each transformed slot to
//                   the leader's barrier
//   8 of the        also the epilogue: after their share of a unit's last
//   transform warps slot, TMEM -> the 8 coordinates of each (o, i), 32
//                   contiguous bytes of the partials
// The transform is bound by instruction issue and latency, not by shared
// memory: spreading a slot's 64 atoms over all 18 warps but the producer and
// the issuer instead of 10 (the epilogue runs once per unit of ~57 slots)
// shortens a slot's critical path from 7 atoms per warp to 4.
//
// Every mbarrier wait is bounded: on timeout the kernel records a code (with
// this launch's epoch) in the fault words, stops, lets copies in flight land,
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "eqlin_internal.cuh"
#include "tc_host.h"
#include "tc_primitives.cuh"
#include "tc_transforms.cuh"

namespace eqlin {
namespace {

constexpr int kWtThreads = 640;
constexpr int kWtProd = 0;       // TMA producer; TMEM allocation
constexpr int kWtMma = 1;        // MMA issuer (leader CTA)
constexpr int kWtTf0 = 2;        // in-place transform: warps kWtTf0..
constexpr int kWtNumTf = 18;
constexpr int kWtEpi0 = 12;      // the last kWtNumEpi of them also drain TMEM -> partials
constexpr int kWtNumEpi = 8;
static_assert(kWtTf0 + kWtNumTf == kWtThreads / 32, "warp roles cover the CTA");
static_assert(kWtEpi0 + kWtNumEpi == kWtThreads / 32, "epilogue warps are the last transform warps");
static_assert(kWtNumEpi == 8, "two epilogue warps per TMEM lane quarter");

constexpr int kWtTk = 32;                         // tokens per slot
constexpr int kWtKSlices = kWtTk / 16;            // MMA K-steps per slot
constexpr int kWtAtoms = kWtTk / 8;               // 1 KB atoms per box
constexpr int kWtBoxBytes = kWtTk * 128;          // 8 fields x kWtTk tokens
constexpr int kWtHalfBytes = 8 * kWtBoxBytes;     // one tensor's 64 fields
constexpr int kWtStageBytes = 2 * kWtHalfBytes;   // dy, then x
constexpr int kWtStages = 3;
constexpr int kWtUnroll = 2;                      // atoms a transform warp handles per pass
constexpr int kWtOTile = 128;                     // output fields per tile (64 per CTA)
constexpr int kWtITile = 128;                     // input fields per tile
constexpr int kWtSub = 64;                        // input fields per subtile (32 per CTA)
constexpr uint32_t kWtTmemCols = 512;
constexpr int kWtCtrlBytes = 256;
constexpr int kWtSmem = 1024 + kWtStages * kWtStageBytes + kWtCtrlBytes;
constexpr uint64_t kWtWaitLimitNs = 2000000000ull;
constexpr uint32_t kWtSleepNs = 128;
// Token splits are sized for this many CTA pairs.  Units are dealt out
// round-robin (unit u to pair u mod P); P prime makes every pair visit every
// tile of a layer with at most 4 tiles once per P units, so tiles of
// different cost (a ragged last tile) spread evenly.
constexpr int kWtPairs = 73;
static_assert(kWtSmem <= 232448, "shared memory");

// One MMA of a K-step: A = DY coordinate ca, B = X coordinate cb, into TMEM
// coordinate group g, B negated if neg.  (A switch rather than a table keeps
// it out of local memory.)
struct WtMma {
  int ca, cb, g, neg;
};
constexpr int kWtMmas = 14;
__host__ __device__ constexpr WtMma wt_mma(int f) {
  switch (f) {
    case 0: return {0, 0, 0, 0};    // C_0 += DY_0 . X_0
    case 1: return {7, 7, 7, 0};    // C_4 += DY_4 . X_4
    case 2: return {1, 1, 1, 0};    // Re C_1 += Re DY_1 . Re X_1
    case 3: return {2, 2, 1, 0};    // Re C_1 += Im DY_1 . Im X_1
    case 4: return {2, 1, 2, 0};    // Im C_1 += Im DY_1 . Re X_1
    case 5: return {1, 2, 2, 1};    // Im C_1 -= Re DY_1 . Im X_1
    case 6: return {3, 3, 3, 0};    // bin 2: Re = c3, Im = c4
    case 7: return {4, 4, 3, 0};
    case 8: return {4, 3, 4, 0};
    case 9: return {3, 4, 4, 1};
    case 10: return {5, 5, 5, 0};   // bin 3: Re = c5, Im = c6
    case 11: return {6, 6, 5, 0};
    case 12: return {6, 5, 6, 0};
    case 13: return {5, 6, 6, 1};
    default: return {0, 0, 0, 0};
  }
}

struct WtArgs {
  float *part;           // [S][Cout][Cin][8] fp32
  unsigned int *fault;   // the two fault words (tc::FaultCtx)
  unsigned int epoch;    // this launch's fault epoch
  int64_t T;
  int Cin, Cout;
  int n_it;              // input-field tiles
  int ntile;             // tiles per split
  int units;             // S * ntile
  int tps;               // tokens per split (a multiple of kWtTk)
};

// Epilogue of one unit, run by warp `warp` (kWtEpi0..) of CTA `rank`: TMEM
// lane quarter q4 = warp % 4 holds rows 32 (q4 % 2).. of this CTA, input fields
// of the first (q4 < 2) or second half of each subtile; the two warps of a
// quarter take 16 rows each.  A 16x256b load of group c gives thread t columns
// 2(t%4), 2(t%4)+1 of rows t/4 and t/4 + 8; eight loads (c = 0..7) give it all
// coordinates of 4 (o, i) items, 32 bytes each.  Not inlined, its loops not
// unrolled: the kernel then needs no more than 96 registers without spills.
__device__ __noinline__ void wgrad_epilogue(float *part, int Cout, int Cin, uint32_t tmem_base,
                                            int split, int ot, int it, int nsub, int rank, int warp,
                                            int lane) {
  using namespace tc;
  const int q4 = warp & 3;
  const int h = q4 >> 1;
  const int sub = (warp - kWtEpi0) >> 2;
  const int tq = lane & 3, tr = lane >> 2;
  const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32 + sub * 16) << 16);
  const int o0 = ot * kWtOTile + rank * 64 + (q4 & 1) * 32 + sub * 16 + tr;
#pragma unroll 1
  for (int st = 0; st < nsub; ++st) {
#pragma unroll 1
    for (int fg = 0; fg < 32; fg += 8) {
      uint32_t v[8][4];
#pragma unroll
      for (int c = 0; c < 8; ++c) tmem_ld_16x256b(tb + (uint32_t)(c * 64 + st * 32 + fg), v[c]);
      tmem_wait_ld();
      const int i0 = it * kWtITile + st * kWtSub + h * 32 + fg + 2 * tq;
#pragma unroll
      for (int e = 0; e < 4; ++e) {   // e = 2 (row + 8) + (column + 1)
        const int o = o0 + 8 * (e >> 1), i = i0 + (e & 1);
        if (o < Cout && i < Cin) {
          // two 16-byte stores: the workspace is only 16-byte aligned
          uint4 *dst = reinterpret_cast<uint4 *>(part + (((size_t)split * Cout + o) * Cin + i) * 8);
          dst[0] = make_uint4(v[0][e], v[1][e], v[2][e], v[3][e]);
          dst[1] = make_uint4(v[4][e], v[5][e], v[6][e], v[7][e]);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kWtThreads, 1)
    cyclic8_wgrad_tc_kernel(const __grid_constant__ CUtensorMap map_dy,
                            const __grid_constant__ CUtensorMap map_x, const WtArgs args) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);
  const uint32_t sBar = base + (uint32_t)(kWtStages * kWtStageBytes);
  auto bar_full = [&](int s) { return sBar + 8u * s; };                   // TMA landed (local)
  auto bar_empty = [&](int s) { return sBar + 8u * (kWtStages + s); };    // MMAs done (local)
  auto bar_xf = [&](int s) { return sBar + 8u * (2 * kWtStages + s); };   // transformed
  const uint32_t bar_acc_full = sBar + 8u * (3 * kWtStages);              // local
  const uint32_t bar_acc_empty = sBar + 8u * (3 * kWtStages + 1);         // leader
  const uint32_t tmem_slot = sBar + 8u * (3 * kWtStages + 2);
  static_assert(8 * (3 * kWtStages + 2) + 4 <= kWtCtrlBytes, "control block");
  volatile uint32_t *tmem_slot_ptr = reinterpret_cast<volatile uint32_t *>(gbase + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const FaultCtx fault{args.fault, args.epoch};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWtStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
      mbar_init(bar_xf(s), kWtNumTf + (leader ? 1 : 0));   // this CTA's transform warps (+ the peer's forwarder)
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_empty, 2 * kWtNumEpi);
    fence_mbarrier_init_cluster();
  }
  if (warp == kWtProd) tmem_alloc_pair(tmem_slot, kWtTmemCols);
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();
  tcgen05_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;

  const int64_t T = args.T;
  const int nunits = args.units > pair ? (args.units - pair + npairs - 1) / npairs : 0;
  // unit u = pair + n * npairs: split u / ntile, tile u % ntile = (ot, it)
  auto unit_split = [&](int n) { return (pair + n * npairs) / args.ntile; };
  auto unit_tile = [&](int n) { return (pair + n * npairs) % args.ntile; };
  auto unit_chunks = [&](int n) {
    const int64_t t0 = (int64_t)unit_split(n) * args.tps;
    const int64_t t1 = t0 + args.tps < T ? t0 + args.tps : T;
    return (int)((t1 - t0 + kWtTk - 1) / kWtTk);
  };
  // subtiles of tile `it` with at least one input field
  auto unit_nsub = [&](int n) {
    const int it = unit_tile(n) % args.n_it;
    return args.Cin - it * kWtITile > kWtSub ? 2 : 1;
  };

  if (warp == kWtProd) {
    // ------------------------------------------------------------ producer
    if (elect_one_sync()) {
      prefetch_tensormap(&map_dy);
      prefetch_tensormap(&map_x);
      uint32_t q = 0;   // slot use counter over all units
      bool ok = true;
      for (int n = 0; n < nunits && ok; ++n) {
        const int tile = unit_tile(n);
        const int ot = tile / args.n_it, it = tile % args.n_it;
        const int64_t t0 = (int64_t)unit_split(n) * args.tps;
        const int nch = unit_chunks(n);
        for (int ch = 0; ch < nch; ++ch, ++q) {
          const int s = (int)(q % kWtStages);
          const uint32_t ph = (q / kWtStages) & 1u;
          if (!mbar_wait_bounded(bar_empty(s), ph ^ 1u, fault, FAULT_WAIT_B_EMPTY, kWtWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t slot = base + (uint32_t)(s * kWtStageBytes);
          const int32_t tok = (int32_t)(t0 + (int64_t)ch * kWtTk);
          mbar_arrive_expect_tx(bar_full(s), (uint32_t)kWtStageBytes);
          for (int b = 0; b < 8; ++b) {
            const int fo = ot * kWtOTile + (int)rank * 64 + 8 * b;
            tma_load_2d(slot + (uint32_t)(b * kWtBoxBytes), &map_dy, bar_full(s), fo * 8, tok);
          }
          for (int b = 0; b < 8; ++b) {
            const int fi = it * kWtITile + (b >> 2) * kWtSub + (int)rank * 32 + 8 * (b & 3);
            tma_load_2d(slot + (uint32_t)(kWtHalfBytes + b * kWtBoxBytes), &map_x, bar_full(s),
                        fi * 8, tok);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kWtMma) {
    // ------------------------------------------------------------ MMA issue (leader CTA)
    if (leader) {
      WtMma md[kWtMmas];
      uint32_t acc_first[kWtMmas];   // 1: an earlier MMA of the K-step already wrote the group
#pragma unroll
      for (int f = 0; f < kWtMmas; ++f) {
        md[f] = wt_mma(f);
        acc_first[f] = 0u;
#pragma unroll
        for (int e = 0; e < f; ++e)
          if (wt_mma(e).g == md[f].g) acc_first[f] = 1u;
      }
      // K-major, no swizzle: core matrices 8 field rows x 16 bytes (8 tokens);
      // along K (token blocks) 1 KB apart, along M/N (8-field boxes) one box apart
      const uint64_t d0 = smem_desc_kmajor_noswizzle(base, 1024u, (uint32_t)kWtBoxBytes);
      const uint32_t d_lo = (uint32_t)d0, d_hi = (uint32_t)(d0 >> 32);
      uint32_t q = 0;
      bool ok = true;
      for (int n = 0; n < nunits && ok; ++n) {
        const int nch = unit_chunks(n);
        // N = 64 per subtile holding fields
        const uint32_t idesc = idesc_bf16_f32(128, kWtSub * unit_nsub(n));
        if (!mbar_wait_bounded_warp(bar_acc_empty, ((uint32_t)n & 1u) ^ 1u, fault,
                                    FAULT_WAIT_ACC_EMPTY, kWtWaitLimitNs)) {
          ok = false;
          break;
        }
        tcgen05_fence_after();
        for (int ch = 0; ch < nch; ++ch, ++q) {
          const int s = (int)(q % kWtStages);
          const uint32_t ph = (q / kWtStages) & 1u;
          if (!mbar_wait_bounded_warp(bar_xf(s), ph, fault, FAULT_WAIT_A_FULL, kWtWaitLimitNs)) {
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint32_t slot16 = (uint32_t)(s * kWtStageBytes) >> 4;
          if (elect_one_sync()) {
#pragma unroll 1   // (unrolled, the kernel spills at 112 registers)
            for (int ks = 0; ks < kWtKSlices; ++ks) {
              const uint32_t acc = (ch > 0 || ks > 0) ? 1u : 0u;
              const uint32_t k16 = (uint32_t)(ks * 2 * 1024) >> 4;
              constexpr uint32_t b16 = (uint32_t)kWtHalfBytes >> 4;
#pragma unroll
              for (int f = 0; f < kWtMmas; ++f) {
                const uint32_t a_lo = d_lo + slot16 + k16 + (uint32_t)(md[f].ca * 128 >> 4);
                const uint32_t b_lo = d_lo + slot16 + b16 + k16 + (uint32_t)(md[f].cb * 128 >> 4);
                mma_bf16_pair_w(tmem_base + (uint32_t)(md[f].g * 64), a_lo, d_hi, b_lo, d_hi,
                                idesc | (md[f].neg ? (1u << 14) : 0u), acc | acc_first[f]);
              }
            }
            mma_commit_pair_mc(bar_empty(s), 0x3);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one_sync()) mma_commit_pair_mc(bar_acc_full, 0x3);
        __syncwarp();
      }
    } else {
      // ---------------------------------------------------------- forwarder (peer CTA)
      // The transform warps arrive on their own CTA's xf barrier (release at
      // CTA scope).  This warp waits for the peer CTA's slot to complete and
      // forwards it to the leader's barrier with one cluster-scope release:
      // such a release blocks the arriving warp for about 0.8 us (traces), so
      // one per slot here replaces 18 on the transform warps' critical path
      // (446 us -> 331 us at 160 x 160 fields, T = 131072).
      const uint32_t leader_xf0 = mapa_shared(bar_xf(0), 0);
      uint32_t q = 0;
      bool ok = true;
      for (int n = 0; n < nunits && ok; ++n) {
        const int nch = unit_chunks(n);
        for (int ch = 0; ch < nch; ++ch, ++q) {
          const int s = (int)(q % kWtStages);
          const uint32_t ph = (q / kWtStages) & 1u;
          if (!mbar_wait_bounded_warp(bar_xf(s), ph, fault, FAULT_WAIT_A_FULL, kWtWaitLimitNs)) {
            ok = false;
            break;
          }
          if (elect_one_sync()) mbar_arrive_cluster(leader_xf0 + 8u * (uint32_t)s);
          __syncwarp();
        }
      }
    }
  } else if (warp >= kWtTf0) {
    // ------------------------------------------------------------ in-place transform (+ epilogue)
    // Item j of a slot (j < 8 kWtAtoms: dy, then x): box (j / kWtAtoms) % 8,
    // atom j % kWtAtoms.  Lane (f = lane % 8, p = lane / 8) takes field f of
    // the box and tokens 2p, 2p+1 of the atom.  Boxes wholly past the layer's
    // fields hold TMA's zero fill, whose transform is zero: they are skipped.
    const int tw = warp - kWtTf0;
    const bool epi = warp >= kWtEpi0;
    const int f = lane & 7, p = lane >> 3;
    uint32_t q = 0;
    bool ok = true;
    // this warp's atoms j = tw + kWtNumTf k of a slot: their byte offsets in
    // the slot (with this lane's two token rows) and which hold fields of the
    // layer are fixed for a unit, so they are worked out once per unit
    constexpr int kMyAtoms = (16 * kWtAtoms + kWtNumTf - 1) / kWtNumTf;
    const int r0 = 2 * p, r1 = 2 * p + 1;   // token rows of an atom
    for (int n = 0; n < nunits && ok; ++n) {
      const int tile = unit_tile(n);
      const int ot = tile / args.n_it, it = tile % args.n_it;
      const int nch = unit_chunks(n);
      uint32_t off[kMyAtoms];
      uint32_t live = 0;
#pragma unroll
      for (int k = 0; k < kMyAtoms; ++k) {
        const int j = tw + k * kWtNumTf;
        const int which = j / (8 * kWtAtoms);
        const int b = (j / kWtAtoms) % 8, a = j % kWtAtoms;
        const int field0 = which == 0 ? ot * kWtOTile + (int)rank * 64 + 8 * b
                                      : it * kWtITile + (b >> 2) * kWtSub + (int)rank * 32 + 8 * (b & 3);
        if (j < 16 * kWtAtoms && field0 < (which == 0 ? args.Cout : args.Cin)) live |= 1u << k;
        off[k] = (uint32_t)(which * kWtHalfBytes + b * kWtBoxBytes + a * 1024);
      }
      for (int ch = 0; ch < nch; ++ch, ++q) {
        const int s = (int)(q % kWtStages);
        const uint32_t ph = (q / kWtStages) & 1u;
        if (!mbar_wait_bounded(bar_full(s), ph, fault, FAULT_WAIT_X_FULL, kWtWaitLimitNs,
                               kWtSleepNs)) {
          ok = false;
          break;
        }
        uint8_t *const slot = gbase + (size_t)s * kWtStageBytes;
        // kWtUnroll atoms per pass: their loads are all in flight together, then
        // each is transformed and rewritten in place
#pragma unroll
        for (int k0 = 0; k0 < kMyAtoms; k0 += kWtUnroll) {
          uint4 v[kWtUnroll][2];
#pragma unroll
          for (int u = 0; u < kWtUnroll; ++u) {
            const int k = k0 + u;
            if (k < kMyAtoms && ((live >> k) & 1u)) {
              v[u][0] = *reinterpret_cast<const uint4 *>(slot + off[k] + r0 * 128 + ((f ^ r0) << 4));
              v[u][1] = *reinterpret_cast<const uint4 *>(slot + off[k] + r1 * 128 + ((f ^ r1) << 4));
            }
          }
          __syncwarp();   // these atoms are whole in registers before any is overwritten
#pragma unroll
          for (int u = 0; u < kWtUnroll; ++u) {
            const int k = k0 + u;
            if (k >= kMyAtoms || !((live >> k) & 1u)) continue;
            float2 xv[8], z[8];
            unpack_bf16x8_pair(v[u][0], v[u][1], xv);
            fwd_cyclic8(xv, z);
            uint8_t *const dst = slot + off[k] + f * 16 + p * 4;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint32_t *>(dst + c * 128) = pack_bf16x2(z[c].x, z[c].y);
          }
          __syncwarp();
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_local(bar_xf(s));
      }
      if (!ok || !epi) continue;
      // ---------------------------------------------------------- epilogue of unit n
      // (the other transform warps run ahead into the next unit's slots); a
      // non-inlined call keeps its registers out of the transform loop
      if (!mbar_wait_bounded(bar_acc_full, (uint32_t)n & 1u, fault, FAULT_WAIT_ACC_FULL,
                             kWtWaitLimitNs, kWtSleepNs)) {
        ok = false;
        break;
      }
      tcgen05_fence_after();
      wgrad_epilogue(args.part, args.Cout, args.Cin, tmem_base, unit_split(n), ot, it, unit_nsub(n),
                     (int)rank, warp, lane);
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(bar_acc_empty, 0));
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
  if (warp == kWtProd) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem_base, kWtTmemCols);
  }
}

struct WtDevCache {
  int max_clusters = 0;
  bool attr_set = false;
};
std::mutex g_wt_mu;
WtDevCache g_wt_cache[64];

}  // namespace

// ---------------------------------------------------------------- interface

// At least 8 fields each way: a tensor map's rows are then never narrower
// than one 8-field box.
bool cyclic_wgrad_tc_supported(int64_t T, int N, int Cin, int Cout, int dtype) {
  return dtype == EQLIN_BF16 && N == 8 && Cin >= 8 && Cout >= 8 && T >= 0 &&
         T <= (int64_t)0x7fff0000LL;
}

WgradTcPlan cyclic_wgrad_tc_plan(int64_t T, int Cin, int Cout) {
  WgradTcPlan p;
  p.n_ot = (Cout + kWtOTile - 1) / kWtOTile;
  p.n_it = (Cin + kWtITile - 1) / kWtITile;
  p.ntile = p.n_ot * p.n_it;
  p.splits = 0;
  p.tokens_per_split = kWtTk;
  if (T <= 0) return p;
  const int64_t target = p.ntile <= 4 ? kWtPairs : (4 * kWtPairs + p.ntile - 1) / p.ntile;
  int64_t tps = (T + target - 1) / target;
  tps = (tps + kWtTk - 1) / kWtTk * kWtTk;
  p.tokens_per_split = (int)tps;
  p.splits = (int)((T + tps - 1) / tps);
  return p;
}

int launch_cyclic_wgrad_tc_partials(const void *x, const void *dy, float *part, int64_t T, int Cin,
                                    int Cout, const WgradTcPlan &plan, cudaStream_t s) {
  if (plan.splits <= 0) return EQLIN_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(EQLIN_ERR_CUDA, "cudaGetDevice failed");
  int maxc = 0;
  {
    std::lock_guard<std::mutex> lk(g_wt_mu);
    WtDevCache &dc = g_wt_cache[dev];
    if (!dc.attr_set) {
      cudaError_t e = cudaFuncSetAttribute(cyclic8_wgrad_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kWtSmem);
      if (e != cudaSuccess)
        return set_error(EQLIN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(kWtThreads, 1, 1);
      cfg.dynamicSmemBytes = kWtSmem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int nc = 0;
      e = cudaOccupancyMaxActiveClusters(&nc, cyclic8_wgrad_tc_kernel, &cfg);
      if (e != cudaSuccess || nc <= 0)
        return set_error(EQLIN_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s (n=%d)",
                         cudaGetErrorString(e), nc);
      dc.max_clusters = nc;
      dc.attr_set = true;
    }
    maxc = dc.max_clusters;
  }
  unsigned int *fw = nullptr;
  int rc = fault_word_address(&fw);
  if (rc) return rc;
  CUtensorMap mdy, mx;
  rc = tma_map_2d_bf16(&mdy, dy, (uint64_t)Cout * 8, (uint64_t)T, (uint64_t)Cout * 16, 64, kWtTk, true);
  if (rc) return rc;
  rc = tma_map_2d_bf16(&mx, x, (uint64_t)Cin * 8, (uint64_t)T, (uint64_t)Cin * 16, 64, kWtTk, true);
  if (rc) return rc;
  WtArgs a;
  a.part = part;
  a.fault = fw;
  a.epoch = next_launch_epoch();
  a.T = T;
  a.Cin = Cin;
  a.Cout = Cout;
  a.n_it = plan.n_it;
  a.ntile = plan.ntile;
  a.units = plan.splits * plan.ntile;
  a.tps = plan.tokens_per_split;
  int npairs = kWtPairs < maxc ? kWtPairs : maxc;
  if (npairs > a.units) npairs = a.units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * npairs, 1, 1);
  cfg.blockDim = dim3(kWtThreads, 1, 1);
  cfg.dynamicSmemBytes = kWtSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, cyclic8_wgrad_tc_kernel, mdy, mx, a);
  if (e != cudaSuccess)
    return set_error(EQLIN_ERR_CUDA, "weight-gradient tensor-core launch: %s", cudaGetErrorString(e));
  return check_launch("cyclic8_wgrad_tc_kernel");
}

}  // namespace eqlin
