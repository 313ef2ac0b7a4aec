// Thin inline-PTX wrappers for the sm_100a features the tensor-core kernel
// uses: mbarriers (with bounded waits), TMA tensor loads, cluster addressing,
// tcgen05 TMEM allocation / MMA / commit / loads, and UMMA descriptors.
#pragma once

#include <stdint.h>

namespace eqlin {
namespace tc {

// ------------------------------------------------------------ basic ids

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// ------------------------------------------------------------ mbarriers

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init_cluster() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Arrive (release at CTA scope) on a barrier of this CTA.
__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Arrive (release at cluster scope) on a barrier given by its shared::cluster
// address (from mapa_shared), possibly in the peer CTA.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// Arrive with a CTA-scope release on a barrier given by its shared::cluster
// address: for a barrier of this CTA whose waiters are in this CTA too.
__device__ __forceinline__ void mbar_arrive_cluster_cta(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// Same, relaxed: signals without ordering this thread's earlier memory
// operations (for a consumer whose only hazard is on data already in its
// registers, e.g. TMEM columns after tcgen05.wait::ld).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Fault state of one launch.  `word` points at two device words: word[0]
// keeps the first code any launch recorded (until the host clears it), and
// word[1] the epoch of the latest launch that gave up.  Each launch carries
// its own nonzero epoch, so a wait gives up early only when a wait of the
// same launch ran out; a stale code from an earlier launch stops nothing.
// FaultCtx holds the epoch in a register; FaultCtxSmem reads it from a shared
// memory word the kernel wrote at start (no register held across the kernel).
struct FaultCtx {
  unsigned int *word;
  unsigned int epoch;
  __device__ __forceinline__ unsigned int my_epoch() const { return epoch; }
};
struct FaultCtxSmem {
  unsigned int *word;
  uint32_t epoch_addr;   // shared-memory address of this launch's epoch
  __device__ __forceinline__ unsigned int my_epoch() const {
    unsigned int e;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e) : "r"(epoch_addr) : "memory");
    return e;
  }
};

template <class F>
__device__ __forceinline__ bool fault_raised(const F &f) {
  return *(volatile unsigned int *)(f.word + 1) == f.my_epoch();
}

template <class F>
__device__ __forceinline__ void fault_raise(const F &f, unsigned int code) {
  atomicCAS(f.word, 0u, code);
  // a plain volatile store is enough: the waits poll word[1] with volatile
  // loads, and when two launches give up at once either epoch may stay
  *(volatile unsigned int *)(f.word + 1) = f.my_epoch();
}

// A wait that has lasted this long (far longer than any wait of a healthy
// pipeline) starts to look at the launch's fault state too.  Before that it
// reads only %globaltimer: the fault words live in global memory, and a load
// of them costs a round trip to L2 that, under a full memory pipeline, blinds
// the polling warp for a microsecond or more.
constexpr uint64_t kFaultCheckAfterNs = 20000ull;

// Wait until the phase with the given parity of `bar` completes.  Gives up
// after `limit_ns` (recording `code` and this launch's epoch), or, once the
// wait has lasted kFaultCheckAfterNs, as soon as another wait of the same
// launch has given up; returns false then.  With sleep_ns > 0 the thread
// backs off with __nanosleep between polls, leaving issue slots to the warps
// that share its scheduler (the MMA issuers).
template <class F>
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, const F &fault,
                                                  unsigned int code, uint64_t limit_ns,
                                                  uint32_t sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (sleep_ns) __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0) {
      const uint64_t waited = globaltimer_ns() - t0;
      if (waited > kFaultCheckAfterNs && fault_raised(fault)) return false;
      if (waited > limit_ns) {
        fault_raise(fault, code);
        return false;
      }
    }
  }
}

// Warp-converged wait: every lane polls, and the result is the same on all
// lanes (a lane that gave up makes the whole warp give up).
template <class F>
__device__ __forceinline__ bool mbar_wait_bounded_warp(uint32_t bar, uint32_t parity,
                                                       const F &fault, unsigned int code,
                                                       uint64_t limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, fault, code, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// True on exactly one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one_sync() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------ fences

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tcgen05_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tcgen05_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ------------------------------------------------------------ TMA

__device__ __forceinline__ void prefetch_tensormap(const void *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2-D tiled load into this CTA's shared memory, completion on a local barrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, uint32_t bar, int32_t c0,
                                            int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// 2-D tiled load into this CTA's shared memory whose completion is counted on
// a barrier of the CTA pair's leader (cluster address from mapa_shared).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *map, uint32_t leader_bar,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(map), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}

// L2 prefetch of one box of a 2-D tensor map (no shared memory involved).
__device__ __forceinline__ void tma_prefetch_2d(const void *map, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(c0),
               "r"(c1)
               : "memory");
}

// L2 prefetch of `bytes` contiguous bytes (a multiple of 16, 16-byte aligned).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------ tcgen05

// Allocate `ncols` TMEM columns for the CTA pair; the base address is written
// to shared memory at `dst`.  Issued by one full warp in each CTA of the pair.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 x bf16 -> f32, CTA pair
// (kind::f16).  The 64-bit descriptors are given as (low, high) words; the low
// words carry the start address and leading byte offset, so K-slices and ring
// slots advance with 32-bit adds.
__device__ __forceinline__ void mma_bf16_pair_w(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                                uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"
      "mov.b64 ad, {%1, %2};\n\t"
      "mov.b64 bd, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], ad, bd, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate));
}

// Arrive once on the barrier at the same shared offset in every CTA of `mask`
// when all previously issued tcgen05 operations of this thread complete.
__device__ __forceinline__ void mma_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// 16 lanes x 256 bit: thread t receives columns 2(t%4), 2(t%4)+1 of lanes
// t/4 (r[0], r[1]) and t/4 + 8 (r[2], r[3]), relative to the warp-uniform
// address (lane in bits 16+, column in bits 0-15).
__device__ __forceinline__ void tmem_ld_16x256b(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

// 32-byte global store (dst 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t (&a)[4], const uint32_t (&b)[4]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(a[0]),
               "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, no swizzle ("interleaved"
// canonical layout: 8-row x 16-byte core matrices, rows 16 B apart).
//   lbo: byte distance between the two core matrices along K
//   sbo: byte distance between consecutive 8-row groups along M/N
__device__ __forceinline__ uint64_t smem_desc_kmajor_noswizzle(uint32_t addr, uint32_t lbo,
                                                               uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  // base offset 0, absolute LBO mode 0, layout type 0 (no swizzle)
  return d;
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row x 128-byte
// atoms (1024 B, 1024-aligned), 16-byte chunk c of row r stored at chunk
// position c ^ (r % 8); atoms stacked along M/N every 1024 B.  A K-step of 16
// bf16 elements starting at chunk 2s is addressed by adding 32*s bytes to the
// atom base.
__device__ __forceinline__ uint64_t smem_desc_kmajor_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;              // leading byte offset: unused for swizzled K-major
  d |= (uint64_t)(1024u >> 4) << 32;   // stride byte offset: 8-row atoms 1024 B apart
  d |= (uint64_t)1 << 46;              // descriptor version for sm_100
  d |= (uint64_t)2 << 61;              // layout type: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A/B, f32 accumulator, both
// operands K-major, shape M x N (M = 128 for the pair instruction).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                          // D format f32
         | (1u << 7)                        // A format bf16
         | (1u << 10)                       // B format bf16
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// The same with fp16 A and B (format code 0); A and B always share a type.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                          // D format f32
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

}  // namespace tc
}  // namespace eqlin
