// Manhattan (L1) distance between packed 2-bit codes (ADAMAS long-context sparse
// attention article, lnwmold.com/news/826806, §2.3: tokens are ranked by the L1
// distance of their codes to the query's codes; a smaller distance is better).
//
// The article's own kernel subtracts whole 32-bit words and counts the bits of
// the difference, which is not an L1 over 2-bit fields.  This is an exact L1:
// for codes a = (a1 a0) of the key and b = (b1 b0) of the query,
//     |a - b| low bit  s0 = a0 ^ b0
//     |a - b| high bit s1 = (a1 ^ b1) & ~((a0 ^ b0) & (a0 ^ a1))
// With X = key ^ query on whole words (high bits at odd positions, low bits at
// even ones) and E = (key ^ (key << 1)) restricted to odd positions, the word
//     F = X & ~((X << 1) & E)
// holds |a - b| in each 2-bit field, and the sum of its 16 fields is
// popc(F) + popc(F & 0xAAAAAAAA).  Two words share the second count:
// (Fa & 0xAAAAAAAA) | ((Fb >> 1) & 0x55555555) has the high bits of both.
#pragma once

#include "common.cuh"

namespace adamas {

__device__ __forceinline__ void key_odd_mask(const uint32_t (&k)[kCodeWords], uint32_t (&e)[kCodeWords]) {
#pragma unroll
  for (int w = 0; w < kCodeWords; ++w) e[w] = (k[w] ^ (k[w] << 1)) & 0xAAAAAAAAu;
}

__device__ __forceinline__ uint32_t field_absdiff(uint32_t k, uint32_t q, uint32_t e) {
  const uint32_t x = k ^ q;
  return x & ~((x << 1) & e);
}

// L1 distance of one key code row to one query code row.
__device__ __forceinline__ int l1_distance(const uint32_t (&k)[kCodeWords], const uint32_t (&e)[kCodeWords],
                                           const uint32_t* q) {
  int d = 0;
#pragma unroll
  for (int w = 0; w < kCodeWords; w += 2) {
    const uint32_t fa = field_absdiff(k[w], q[w], e[w]);
    const uint32_t fb = field_absdiff(k[w + 1], q[w + 1], e[w + 1]);
    d += __popc(fa) + __popc(fb) + __popc((fa & 0xAAAAAAAAu) | ((fb >> 1) & 0x55555555u));
  }
  return d;
}

}  // namespace adamas
