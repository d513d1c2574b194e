// Inline-PTX wrappers for kernels that run on clusters of two CTAs sharing every tensor-core
// operation (tcgen05 with cta_group::2): cluster rank and barrier, addresses in the peer CTA,
// remote mbarrier arrivals, TMA loads that signal the leader CTA's barrier, pair MMAs and
// commits that arrive on both CTAs' barriers.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"

namespace isa {

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_warp() {  // whole warp
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
// Arrive on a barrier of either CTA. Default (release, CTA scope) semantics: what the
// barrier hands over is TMEM data, ordered by tcgen05.wait::st and the tcgen05 fences
// around the barrier; a cluster-scope release here measured 1.4x slower for the kernel.
__device__ __forceinline__ void arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void store_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// TMA load into this CTA's shared memory, completion counted on a barrier of the leader CTA.
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Arrive on `bar` in both CTAs once every MMA issued so far is complete.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .b64 da, db;\n\t.reg .pred p;\n\tmov.b64 da, {%1, %5};\n\tmov.b64 db, {%2, %5};\n\t"
      "setp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(acc), "r"(hi)
      : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .b64 db;\n\t.reg .pred p;\n\tmov.b64 db, {%2, %5};\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], db, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(acc), "r"(hi)
      : "memory");
}

// The same three instructions for a converged warp: every lane runs them with the same
// (warp-uniform) operands and elect.sync picks the one lane that issues (as the cta_group::1
// forms in ptx.cuh, and for the same reason).
__device__ __forceinline__ void commit_pair_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}\n" ::"r"(
          smem_addr(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair_warp(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                                 uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .b64 da, db;\n\t.reg .pred p, e;\n\tmov.b64 da, {%1, %5};\n\tmov.b64 db, {%2, %5};\n\t"
      "setp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(acc), "r"(hi)
      : "memory");
}
__device__ __forceinline__ void mma_ts_pair_warp(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                                 uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .b64 db;\n\t.reg .pred p, e;\n\tmov.b64 db, {%2, %5};\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], db, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(acc), "r"(hi)
      : "memory");
}

}  // namespace isa
