// Inline-PTX wrappers for a CTA pair (a cluster of 2 CTAs on the two SMs of
// a TPC) driving tcgen05.mma.cta_group::2: an M = 256 UMMA whose A rows and
// accumulator rows are split over the two CTAs (128 each) and whose B
// columns are split likewise (N/2 each), issued by the even CTA (the leader)
// alone.  Barriers one CTA signals in the other are addressed through the
// shared::cluster window (mapa).  No load here multicasts.
#pragma once

#include "sm100_ptx.cuh"

namespace apb {
namespace pair {

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t n_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// shared::cluster address of the object at `p` (this CTA's shared memory) in
// the shared memory of CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(ptx::smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Arrival (release at cluster scope) on a barrier given by its
// shared::cluster address, in this CTA or the peer.
__device__ __forceinline__ void arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void arrive_expect_tx_remote(uint32_t bar_cluster, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
          bar_cluster),
      "r"(bytes)
      : "memory");
}

// The same without release semantics: for a producer whose arrival publishes
// no memory writes of its own (the bytes of its TMA loads are counted by the
// barrier itself), so the thread is not held until its earlier accesses are
// visible across the cluster.
__device__ __forceinline__ void arrive_expect_tx_relaxed(uint32_t bar_cluster, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
          bar_cluster),
      "r"(bytes)
      : "memory");
}

// Phase wait with acquire at cluster scope (the arrivals come from both CTAs).
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
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

__device__ __forceinline__ bool test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Polls without suspending: for the UMMA issuer, whose reaction time is on
// the critical path.
__device__ __forceinline__ bool spin_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                     const volatile uint32_t* abort,
                                                     uint64_t limit_ns) {
  const uint32_t a = ptx::smem_u32(bar);
  if (test_wait_cluster(a, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (test_wait_cluster(a, parity)) return true;
    if (*abort != 0u) return false;
    if (ptx::globaltimer() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ bool wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                     const volatile uint32_t* abort,
                                                     uint64_t limit_ns) {
  const uint32_t a = ptx::smem_u32(bar);
  if (try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (try_wait_cluster(a, parity)) return true;
    if (*abort != 0u) return false;
    if (ptx::globaltimer() - t0 > limit_ns) return false;
  }
}

// TMA tile load into this CTA's shared memory whose completion bytes are
// counted on a barrier that may live in the peer CTA (the leader's).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint32_t bar_cluster,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(ptx::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   ptx::smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T over the pair, bf16 in, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One arrival on the barrier at `bar_cluster` (either CTA) once every UMMA
// the leader issued before it has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar_cluster) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          bar_cluster)
      : "memory");
}

}  // namespace pair
}  // namespace apb
