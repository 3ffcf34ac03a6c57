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
