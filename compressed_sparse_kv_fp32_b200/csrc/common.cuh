// Shared device helpers for the ADAMAS sm_100a kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace adamas {

constexpr int kDim = 128;            // head dimension (one bucketing group)
constexpr int kCodeBytes = kDim / 4; // packed 2-bit codes per vector
constexpr int kCodeWords = kCodeBytes / 4;
constexpr int kBins = 3 * kDim + 1;  // L1 distance of 2-bit codes lies in [0, 384]
constexpr int kMaxGroup = 8;         // query heads per kv head handled by the kernels
constexpr int kMaxBatch = 1024;

// Bits of the device error word (mirrors ADAMAS_DEVERR_* in adamas.h).
constexpr uint32_t kErrSeqLen = 0x1u;
constexpr uint32_t kErrTimeout = 0x2u;
constexpr uint32_t kErrInternal = 0x4u;

// RN_fp32(1/sqrt(128)), bit pattern 0x3DB504F3: the rotation's normalisation.
__device__ __forceinline__ float hadamard_norm() { return __uint_as_float(0x3DB504F3u); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 32-byte streaming load (one packed code row), bypassing L1 allocation.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------- bulk async copies (no multicast)
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Explicit shared-memory accesses at a shared-window address (ordered like the
// barriers around them).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
// Shared-window address of the same location in cluster block `rank`, and a
// relaxed cluster-scope load from such an address (several may be in flight).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_relaxed_cluster(uint32_t a) {
  uint32_t v;
  asm volatile("ld.relaxed.cluster.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
// Split cluster barrier: arrive (release: this thread's earlier writes become
// visible to the cluster) and wait (acquire).  Every thread alternates the two.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }

__device__ __forceinline__ void sts16(uint32_t a, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}

// Programmatic dependent launch: allow the next kernel of the stream to be
// scheduled, and wait until the kernels before this one have completed and
// their memory is visible (returns at once when the launch did not opt in).
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// One global -> shared bulk copy (16-byte aligned addresses, size a multiple of 16)
// whose completion is counted in bytes on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_gpu64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long atom_add_acqrel_gpu64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

__device__ __forceinline__ void red_add_release_gpu64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// 16-byte global -> shared copy through the L2 (cp.async, completion by wait_group).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bring the 128-byte line holding `p` into L2.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
}

// Bring the 128-byte line holding `p` into L2, to be kept there preferentially.
__device__ __forceinline__ void prefetch_l2_keep(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p) : "memory");
}

// Bounded wait for the phase with the given parity of `bar` to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
  const uint32_t a = smem_addr(bar);
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ uint32_t lop3_xor_and(uint32_t a, uint32_t b, uint32_t c) {
  // (a ^ b) & c
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x28;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t lop3_xor_andnot(uint32_t a, uint32_t b, uint32_t c) {
  // (a ^ b) & ~c
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x14;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Unit x of a range [0, total) split evenly over S blocks: block s owns
// [s*total/S, (s+1)*total/S).  Returns the owner of x (0 <= x < total).
__device__ __forceinline__ int owner_of(int64_t x, int64_t total, int S) {
  return (int)(((x + 1) * (int64_t)S - 1) / total);
}
__device__ __forceinline__ int64_t range_begin(int s, int64_t total, int S) {
  return ((int64_t)s * total) / S;
}

}  // namespace adamas
