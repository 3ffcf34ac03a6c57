// Manhattan (L1) distance between packed 2-bit codes (ADAMAS long-context sparse
// attention article, lnwmold.com/news/826806, §2.3: tokens are ranked by the L1
// distance of their codes to the query's codes; a smaller distance is better).
//
// The article's own kernel subtracts whole 32-bit words and counts the bits of
// the difference, which is not an L1 over 2-bit fields.  This is an exact L1.
// For a key code a = (a1 a0) and a query code b = (b1 b0):
//     low bit of |a - b|   = a0 ^ b0
//     high bit of |a - b|  = (a1 ^ b1) & ((a0 ^ b1) | [b0 == b1])
// (b = 0 or 3: |a - b| >= 2 exactly when a1 != b1; b = 1: only for a = 3;
// b = 2: only for a = 0).  On whole words, with the high bits at odd positions:
//     F = (k ^ q) & (((k << 1) ^ q) | m),   m = odd bits [b0 == b1] | 0x55555555
// holds |a - b| in each 2-bit field.  The query is fixed for a whole scan, so m
// is computed once per query word and each key word costs one shift (shared by
// every query head) and two three-input logic operations per query head.  The
// sum of the 16 fields of F is popc(F) + popc(F & 0xAAAAAAAA); two words share
// the second count: (Fa & 0xAAAAAAAA) | ((Fb >> 1) & 0x55555555) has the high
// bits of both.
#pragma once

#include "common.cuh"

namespace adamas {

// Mask of one packed query word (see the file comment).
__device__ __forceinline__ uint32_t query_mask(uint32_t q) {
  return (~((q << 1) ^ q) & 0xAAAAAAAAu) | 0x55555555u;
}

// |a - b| in every 2-bit field; k1 = k << 1.
__device__ __forceinline__ uint32_t field_absdiff(uint32_t k, uint32_t k1, uint32_t q, uint32_t m) {
  return (k ^ q) & ((k1 ^ q) | m);
}

__device__ __forceinline__ void key_shift(const uint32_t (&k)[kCodeWords], uint32_t (&k1)[kCodeWords]) {
#pragma unroll
  for (int w = 0; w < kCodeWords; ++w) k1[w] = k[w] << 1;
}

// L1 distance of one key code row (k, k1 = k << 1) to one query code row (q, m).
__device__ __forceinline__ int l1_distance(const uint32_t (&k)[kCodeWords], const uint32_t (&k1)[kCodeWords],
                                           const uint32_t (&q)[kCodeWords], const uint32_t (&m)[kCodeWords]) {
  int d = 0;
#pragma unroll
  for (int w = 0; w < kCodeWords; w += 2) {
    const uint32_t fa = field_absdiff(k[w], k1[w], q[w], m[w]);
    const uint32_t fb = field_absdiff(k[w + 1], k1[w + 1], q[w + 1], m[w + 1]);
    d += __popc(fa) + __popc(fb) + __popc((fa & 0xAAAAAAAAu) | ((fb >> 1) & 0x55555555u));
  }
  return d;
}

}  // namespace adamas
