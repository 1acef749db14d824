// sm100_pair_ptx.cuh -- inline-PTX wrappers for kernels whose tensor-core work is shared
// by a pair of CTAs (a cluster of two, tcgen05 ".cta_group::2"): the pair's MMA computes
// an M=256 tile whose A rows and B columns are split between the two CTAs' shared
// memories and whose accumulator rows are split between their tensor memories.
//
// Every tcgen05 instruction of such a kernel uses cta_group::2; the cta_group::1
// wrappers of sm100_ptx.cuh must not be mixed into it.
#pragma once

#include "sm100_ptx.cuh"

namespace dsmoe {
namespace pair {

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs; orders earlier shared-memory writes (and mbarrier inits)
// before everything after the barrier, cluster-wide.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the object at shared::cta address `saddr` in CTA `rank`.
__device__ __forceinline__ uint32_t map_to(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t caddr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t caddr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
  return v;
}

// Arrive on an mbarrier that may live in the other CTA of the pair. Default (CTA-scope)
// release: what it orders for the other CTA is tensor-memory reads, which the caller
// completes (tcgen05.wait::ld) and fences (tcgen05.fence::before_thread_sync) first;
// a cluster-scope release would also wait for this thread's earlier global stores.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// try_wait for barriers that the other CTA (its copies, its arrivals or the pair's MMA
// commits) completes; default acquire semantics, as for the CTA's own barriers.
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait (see mbar_wait_bounded) on such a barrier.
__device__ __forceinline__ bool mbar_wait_bounded_cl(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                     volatile int* abort_flag) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

// Whole-warp bounded wait with back-off (see mbar_wait_warp_sleepy) on such a barrier.
__device__ __forceinline__ bool mbar_wait_warp_sleepy_cl(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                         volatile int* abort_flag) {
  uint32_t ok = 1;
  if ((threadIdx.x & 31) == 0) {
    if (!mbar_try_wait_cl(bar, parity)) {
      const uint64_t t0 = global_timer_ns();
      uint32_t sleep_ns = 32;
      for (;;) {
        __nanosleep(sleep_ns);
        if (mbar_try_wait_cl(bar, parity)) break;
        if (sleep_ns < 512) sleep_ns <<= 1;
        if (*abort_flag || global_timer_ns() - t0 > limit_ns) {
          ok = 0;
          break;
        }
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) (void)mbar_try_wait_cl(bar, parity);
  return ok != 0;
}

// TMA tiled loads into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar_caddr` is a shared::cluster address). No
// multicast: each CTA loads only its own part of the operands.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_caddr, int32_t c0,
                                                 int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_caddr), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_caddr, int32_t c0,
                                                 int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_caddr), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// TMEM allocation shared by the pair: one warp with the same warp index in each CTA
// executes it; both receive the same base address.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// The pair's MMA, issued by one thread of the even CTA: D[256 x N] (+)= A[256 x 16] *
// B[N x 16]^T. A rows 0..127 and B columns 0..N/2-1 come from the even CTA's shared
// memory, A rows 128..255 and B columns N/2..N-1 from the odd CTA's, at the same
// addresses; D rows 0..127 land in the even CTA's TMEM and rows 128..255 in the odd's.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at the same offset in every CTA of `cta_mask` once all earlier
// MMAs of this thread have completed.
__device__ __forceinline__ void mma_commit_both(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(cta_mask)
      : "memory");
}

// The same, on this CTA's barrier only.
__device__ __forceinline__ void mma_commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

}  // namespace pair
}  // namespace dsmoe
