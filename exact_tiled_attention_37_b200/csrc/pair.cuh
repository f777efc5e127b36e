// Inline-PTX primitives for kernels whose CTAs work in pairs (a cluster of
// two CTAs on the two SMs of one TPC) and issue tcgen05 products with
// .cta_group::2: one M = 256 product whose rows 0-127 live in the even CTA
// and rows 128-255 in the odd one, B split along N between the two shared
// memories, accumulators in each CTA's own tensor memory.
//
// Rules every pair kernel here follows:
//  * every tcgen05 instruction of the kernel (alloc, relinquish, dealloc,
//    mma, commit) uses .cta_group::2; tcgen05.ld / st / wait / fence have
//    no CTA-group qualifier;
//  * only the even CTA (rank 0, the leader) issues products and commits; a
//    commit that both CTAs' barriers must see is one instruction with a
//    two-CTA mask (a completion signal, no data);
//  * TMA loads never broadcast: each CTA loads its own half of an operand
//    from this GPU's global memory into its own shared memory and reports
//    the bytes to the leader's barrier (.cta_group::2 form);
//  * waits on a barrier that another CTA arrives on use cluster-scope
//    acquire, and every wait is bounded (PairWaiter).
#pragma once

#include "ptx.cuh"

namespace eta {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// All threads of both CTAs: release this CTA's prior writes (barrier inits
// included) to the cluster and acquire the other CTA's.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on a barrier of any CTA of the cluster (cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded waits with cluster-scope acquire (the Waiter protocol of ptx.cuh:
// give up after the limit, record where in the status word, raise this CTA's
// abort flag).
struct PairWaiter {
  volatile uint32_t* abort;
  int* status;
  uint64_t limit_ns;

  __device__ __forceinline__ bool aborted() const { return *abort != 0; }

  __device__ __forceinline__ void fail(int where) const {
    *abort = 1u;
    if (atomicCAS(status, 0, kErrDeviceTimeout) == 0) {
      status[1] = where;
      status[2] = blockIdx.x;
      status[3] = blockIdx.y;
    }
  }

  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, int where) const {
    if (mbar_try_wait_cl(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      if (mbar_try_wait_cl(bar, parity)) return true;
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        fail(where);
        return false;
      }
    }
  }

  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, int where) const {
    const bool ok = wait(bar, parity, where);
    return __all_sync(0xffffffffu, ok);
  }

  // Waits even after an abort (for copies or products this CTA started).
  __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity, int where) const {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cl(bar, parity)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        fail(where);
        return false;
      }
    }
    return true;
  }
};

// 5-D tiled load into this CTA's shared memory whose completion (bytes) is
// reported to `cl_bar`, a barrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_5d_pair(uint32_t dst, const CUtensorMap* m,
                                                 uint32_t cl_bar, int c0, int c1, int c2, int c3,
                                                 int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(cl_bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// Tensor memory for both CTAs of the pair (issued by the same warp of each).
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// M = 256 products over the pair (leader CTA only): A rows from each CTA's
// own operand, B columns split between the two CTAs' shared memories.
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `cl_bar` (a barrier of either CTA, cluster address) when
// every pair product this thread issued so far is complete.
__device__ __forceinline__ void mma_commit_pair(uint32_t cl_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cl_bar)
               : "memory");
}

// The same arrival on the barrier at offset `bar` in each CTA of `cta_mask`
// (bit r = cluster rank r), with one instruction: an arrive signal for
// several CTAs, not a data copy.  A commit costs the tensor pipe about as
// much as a short product, so pair kernels signal both CTAs with one.
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

}  // namespace eta
