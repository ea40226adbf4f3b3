// Thread-block-cluster helpers shared by the clustered layer kernels: cluster
// rank and index, the cluster-wide barrier, addresses in another CTA's shared
// memory and 16-byte stores into it that complete on its mbarrier, plus the
// named barrier of a kernel's 128 epilogue threads. Inline PTX only.
#pragma once

#include "common.cuh"

namespace df {
namespace cl {

// Named barrier 1 over a kernel's N epilogue threads (whole warps).
template <int N = 128>
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

// The same barrier, ANDing a predicate over the epilogue threads, so that a
// wait which gave up in one thread stops all of them together.
template <int N = 128>
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(N)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// All threads of all CTAs of the cluster (each warp converged).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The address of this CTA's shared-memory location `addr` in cluster rank `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// 16 bytes into another CTA's shared memory, counted (complete_tx) on its
// mbarrier `rbar` (a shared::cluster address from map_rank).
__device__ __forceinline__ void st_async16(uint32_t raddr, float a, float b, float c, float d,
                                           uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, "
      "[%5];" ::"r"(raddr),
      "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(__float_as_uint(c)),
      "r"(__float_as_uint(d)), "r"(rbar)
      : "memory");
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// this CTA's shared memory into another CTA's (dst, rbar: shared::cluster
// addresses from map_rank), counted (complete_tx) on its mbarrier. The source
// must have been made visible to the async proxy (fence.proxy.async) first.
__device__ __forceinline__ void bulk_s2cluster(uint32_t dst, const void* src, uint32_t bytes,
                                               uint32_t rbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(dst),
      "r"(smem_u32(src)), "r"(bytes), "r"(rbar)
      : "memory");
}

// Receive slot of sender s in owner o's buffer (0..2) in a 4-CTA cluster.
__device__ __forceinline__ uint32_t recv_slot(uint32_t s, uint32_t o) {
  return (s - o - 1u) & 3u;
}

}  // namespace cl
}  // namespace df
