// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor loads,
// tcgen05 (tensor memory + 5th-generation MMA), bounded waits and the status word.
// Written from the PTX ISA's descriptions of these instructions.  No cluster
// multicast form of any load appears anywhere in this library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// ----------------------------------------------------------------------------------
// Device status word: 0 = fine.  A bounded wait that expires stores a code here.
// ----------------------------------------------------------------------------------
__device__ int g_status;

enum : int { kStatusTimeout = 1, kStatusBadLengths = 2 };

__device__ __forceinline__ void record_status(int code, int where) {
  atomicCAS(&g_status, 0, (code << 16) | (where & 0xffff));
}

__device__ __forceinline__ void record_timeout(int where) { record_status(kStatusTimeout, where); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// A wait gives up after this long (ns).  Kernels here finish in milliseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false (and
// records `where` in the status word) if it did not within kWaitLimitNs, or if
// *abort became non-zero meanwhile (another role already gave up).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort && *abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_timeout(where);
        if (abort) *abort = 1;
        return false;
      }
    }
  }
}

// One arrival for the whole warp (all 32 lanes execute it; elect.sync picks the lane).
__device__ __forceinline__ void mbar_arrive_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
      " @e mbarrier.arrive.shared::cta.b64 _, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait by every lane of a warp, with one answer for the whole warp.  Each poll
// is a warp vote and every branch depends only on votes, so the warp never diverges:
// an already-completed phase costs one poll and one vote (a per-lane early return
// would make the compiler split and re-converge the warp around every wait).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity,
                                               volatile int* abort, int where) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 255u) == 0) {
      if (__any_sync(0xffffffffu, abort != nullptr && *abort != 0)) return false;
      if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) {
        if ((threadIdx.x & 31) == 0) {
          record_timeout(where);
          if (abort) *abort = 1;
        }
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------------
// TMA (tensor loads, no multicast)
// ----------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load into shared memory; completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Plain bulk copy global -> shared memory (no tensor map, no multicast); both addresses
// 16-byte aligned, bytes a multiple of 16; completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ----------------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads/stores, fences
// ----------------------------------------------------------------------------------
// Whole warp: allocate `ncols` TMEM columns, base address written to *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// tcgen05.mma (D[tmem] (+)= A * B, A from a shared-memory descriptor or tensor memory, B
// from a shared-memory descriptor) and tcgen05.commit (arrive once on `bar` when every
// tcgen05 op issued so far has completed), in warp-wide form: all 32 lanes execute them
// with the same operands and elect.sync picks the one lane that issues.  Keeping the
// issuing code warp-uniform (no lane-0 branch) lets the operands stay on the uniform
// datapath, so an MMA costs a few issue slots even while the softmax warps on the same
// scheduler issue every cycle.
//
// Batches of k-steps in one asm block, one elect.sync per batch (fewer instructions for
// the issuing warp, whose scheduler it shares with two busy softmax warps).  A descriptor
// holds the shared-memory address >> 4 in its low 14 bits; addresses stay below 256 KB, so
// stepping a descriptor is a plain add on it.
//   mma_ss_x4: 4 k-steps of 16 elements along a 128-byte swizzled row: both descriptors
//              advance 32 bytes per step; the first step accumulates iff acc_first.
__device__ __forceinline__ void mma_ss_x4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r;\n .reg .b64 a, b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      " add.s64 a, %1, 2;\n add.s64 b, %2, 2;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 4;\n add.s64 b, %2, 4;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 6;\n add.s64 b, %2, 6;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
//   mma_ts_x2: 2 k-steps with A in tensor memory (16 keys = 8 columns of 16-bit pairs per
//              step) and B stepping 16 rows of 128 bytes (2048 bytes) per step.
__device__ __forceinline__ void mma_ts_x2(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %2, 128;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
//   mma_ts_x6: 6 such k-steps.
__device__ __forceinline__ void mma_ts_x6(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %2, 128;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 16;\n add.s64 b, %2, 256;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 24;\n add.s64 b, %2, 384;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 32;\n add.s64 b, %2, 512;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 40;\n add.s64 b, %2, 640;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n"
      ::"r"(smem_u32(bar)) : "memory");
}

// Warp-wide: 32 lanes x 32 consecutive 32-bit columns; thread t gets lane (base+t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 16 columns variant (for 64-column P halves).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// tcgen05.wait::ld that also names the 32 registers a preceding tmem_ld32 filled, so no
// use of them can be scheduled above the wait (the load writes them asynchronously).
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                 "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                 "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                 "+r"(r[31])
               :: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs whose tensor cores run one product together).
// Written from the PTX ISA's descriptions; the pair forms are used by the pair kernel only
// (a kernel uses one cta_group throughout).  Tensor-memory addresses and shared-memory
// descriptors name the same columns / offsets in both CTAs.
// ----------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// One arrival on an mbarrier of another CTA of the cluster.  The default (CTA-scope) release:
// what it signals is tensor-memory data ordered by tcgen05.wait / tcgen05.fence before it;
// the cluster-scope release measured about 1500 cycles per arrival here.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 4-D tiled load into this CTA's shared memory whose completion (bytes) is counted on an
// mbarrier of either CTA of the pair (bar: a shared::cluster address); no multicast.
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded waits (as mbar_wait / mbar_wait_warp) with acquire at cluster scope, for barriers
// that arrivals from the peer CTA or the pair's commits complete.
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort, int where) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort && *abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_timeout(where);
        if (abort) *abort = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait_warp_cl(uint64_t* bar, uint32_t parity, volatile int* abort, int where) {
  if (__all_sync(0xffffffffu, mbar_try_wait_cl(bar, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait_cl(bar, parity))) return true;
    if ((it & 255u) == 0) {
      if (__any_sync(0xffffffffu, abort != nullptr && *abort != 0)) return false;
      if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) {
        if ((threadIdx.x & 31) == 0) {
          record_timeout(where);
          if (abort) *abort = 1;
        }
        return false;
      }
    }
  }
}
// Every thread of both CTAs: arrive and wait at the cluster barrier (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Pair tensor memory: one warp of each CTA (the same warp index in both) allocates the same
// columns in both CTAs' tensor memory; the same warps free them.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair products, issued by the leader CTA: D rows 0-127 in the leader's tensor memory, rows
// 128-255 in the peer's; each CTA supplies its own A rows and half of B (N / 2) at the same
// shared-memory offsets.  x4: 4 k-steps of 16 elements along a 128-byte swizzled row (both
// descriptors advance 32 bytes); ts_x4: 4 k-steps with A (16-bit P) in tensor memory, 8
// columns per step, B stepping 16 rows of 128 bytes.
__device__ __forceinline__ void mma_pair_ss_x4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r;\n .reg .b64 a, b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
      " add.s64 a, %1, 2;\n add.s64 b, %2, 2;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 4;\n add.s64 b, %2, 4;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 6;\n add.s64 b, %2, 6;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
//   ss_x8: 8 k-steps over two 128-byte chunks of both operands (chunk strides a_chunk and
//          b_chunk, in descriptor units of 16 bytes); the first step accumulates iff acc_first.
__device__ __forceinline__ void mma_pair_ss_x8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t acc_first, uint32_t a_chunk, uint32_t b_chunk) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r;\n .reg .b64 a, b, a1, b1;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
      " add.s64 a, %1, 2;\n add.s64 b, %2, 2;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 4;\n add.s64 b, %2, 4;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, %1, 6;\n add.s64 b, %2, 6;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " cvt.u64.u32 a1, %6;\n cvt.u64.u32 b1, %7;\n add.s64 a1, %1, a1;\n add.s64 b1, %2, b1;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a1, b1, %3, q;\n"
      " add.s64 a, a1, 2;\n add.s64 b, b1, 2;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, a1, 4;\n add.s64 b, b1, 4;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n"
      " add.s64 a, a1, 6;\n add.s64 b, b1, 6;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %3, q;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u), "r"(a_chunk), "r"(b_chunk)
      : "memory");
}
//   ts_x8: 8 k-steps with A (16-bit P) in tensor memory at two column bases (keys 0-63 at a0,
//          keys 64-127 at a1, 8 columns per step), B stepping 16 rows of 128 bytes.
__device__ __forceinline__ void mma_pair_ts_x8(uint32_t d_tmem, uint32_t a0, uint32_t a1, uint64_t b_desc,
                                               uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %5, 0;\n setp.ne.b32 q, %6, 0;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %3, %4, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %3, 128;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n"
      " add.u32 a, %1, 16;\n add.s64 b, %3, 256;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n"
      " add.u32 a, %1, 24;\n add.s64 b, %3, 384;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n"
      " add.s64 b, %3, 512;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [%2], b, %4, q;\n"
      " add.u32 a, %2, 8;\n add.s64 b, %3, 640;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n"
      " add.u32 a, %2, 16;\n add.s64 b, %3, 768;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n"
      " add.u32 a, %2, 24;\n add.s64 b, %3, 896;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %4, q;\n}\n"
      ::"r"(d_tmem), "r"(a0), "r"(a1), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
__device__ __forceinline__ void mma_pair_ts_x4(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %2, 128;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 16;\n add.s64 b, %2, 256;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 24;\n add.s64 b, %2, 384;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], [a], b, %3, q;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
// Commit of the pair's products so far: one arrival on the mbarrier at this offset in each
// CTA of the pair (mask 0b11) once they have completed.
__device__ __forceinline__ void mma_commit_pair_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 r;\n .reg .b16 m;\n elect.sync r|e, 0xffffffff;\n mov.b16 m, 3;\n"
      " @e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n}\n"
      ::"r"(smem_u32(bar)) : "memory");
}

// ----------------------------------------------------------------------------------
// UMMA descriptors (tcgen05 shared-memory matrix descriptor and instruction descriptor)
// ----------------------------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
//   bits  0-13 start address >> 4      bits 16-29 leading byte offset >> 4
//   bits 32-45 stride byte offset >> 4 bits 46-47 version (1)
//   bits 49-51 base offset (0: atoms 1024-B aligned)   bit 52 LBO mode (0)
//   bits 61-63 layout: 2 = 128-byte swizzle
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3fff) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3fff) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with fp32 accumulation.
//   bits 4-5 D format (1 = f32); 7-9 A format, 10-12 B format (0 = f16, 1 = bf16);
//   bit 15 A major, bit 16 B major (0 = K-major, 1 = MN-major);
//   bits 17-22 N >> 3; bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16(int bf16, int M, int N, int a_mn_major,
                                                 int b_mn_major) {
  return (1u << 4) | ((uint32_t)bf16 << 7) | ((uint32_t)bf16 << 10) |
         ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Warpgroup-wide register reallocation (all 128 threads of the warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ----------------------------------------------------------------------------------
// small math helpers
// ----------------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pair of fp32 values in one 64-bit register (sm_100 f32x2 arithmetic).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack_f2(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack_f2(f32x2 v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f32x2 fma_f2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 add_f2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max of three fp32 values in one instruction (sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

}  // namespace sa
