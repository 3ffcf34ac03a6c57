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
constexpr uint32_t kErrTable = 0x8u;

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
// whose completion is counted in bytes on `bar`.  The source is read once, so its
// lines are marked first to go from L2 (they should not push out data that is read
// again, like the K/V rows of the gather).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "{\n .reg .b64 pol;\n createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n"
      " cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], pol;\n}" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity of `bar` to complete, for at most about
// `limit_ns` nanoseconds of the global timer (checked every 128 polls; at most 2^26
// polls in any case).  Returns false when it gives up.
__device__ __forceinline__ bool mbar_wait_timed(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_addr(bar);
  uint64_t t_end = 0;
  for (uint32_t i = 0; i < (1u << 26); ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 127u) == 127u) {
      const uint64_t now = global_ns();
      if (t_end == 0) t_end = now + limit_ns;
      else if (now > t_end) return false;
    }
  }
  return false;
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

}  // namespace adamas
