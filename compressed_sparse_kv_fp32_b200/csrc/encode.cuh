// Hadamard rotation + 2-bit dynamic bucketing + packing of one 128-dim vector
// (ADAMAS long-context sparse attention article, lnwmold.com/news/826806:
// §2.1 Hadamard transform, §2.2 dynamic bucketing, §3.1 packed code cache).
//
// Every element goes through the same operations in the same order as the
// Sylvester-order butterfly y = H x / sqrt(128): stage widths h = 1, 2, ..., 64,
// at each stage the pair (x[j], x[j+h]) with bit h of j clear becomes
// (x[j] + x[j+h], x[j] - x[j+h]) in fp32 with round-to-nearest, and at the end
// every element is multiplied once by RN(1/sqrt(128)).  No multiply-add is
// fused, so the rotated values -- and therefore the codes -- are reproducible
// bit for bit by any implementation that keeps this order.
//
// Bucketing: m = max |y_i|, thresholds t0 = -m/2, t1 = 0, t2 = +m/2, code
// 0 if y < t0, 1 if y < t1, 2 if y < t2, else 3, computed as
// 3 - [y < t0] - [y < t1] - [y < t2] (the thresholds are ordered).
// Packing: byte j = c[4j] << 6 | c[4j+1] << 4 | c[4j+2] << 2 | c[4j+3].
#pragma once

#include "common.cuh"

namespace adamas {

__device__ __forceinline__ uint32_t code_of(float y, float t0, float t2) {
  return 3u - (uint32_t)(y < t0) - (uint32_t)(y < 0.0f) - (uint32_t)(y < t2);
}

// ---------------------------------------------------------------- one vector per thread
// v: the 128 elements in registers (constant indices only).
template <int H>
__device__ __forceinline__ void fwht_stage(float (&v)[kDim]) {
#pragma unroll
  for (int i = 0; i < kDim; i += 2 * H) {
#pragma unroll
    for (int j = i; j < i + H; ++j) {
      const float a = v[j], b = v[j + H];
      v[j] = __fadd_rn(a, b);
      v[j + H] = __fsub_rn(a, b);
    }
  }
}

__device__ __forceinline__ void fwht128_thread(float (&v)[kDim]) {
  fwht_stage<1>(v);
  fwht_stage<2>(v);
  fwht_stage<4>(v);
  fwht_stage<8>(v);
  fwht_stage<16>(v);
  fwht_stage<32>(v);
  fwht_stage<64>(v);
  const float c = hadamard_norm();
#pragma unroll
  for (int j = 0; j < kDim; ++j) v[j] = __fmul_rn(v[j], c);
}

// Rotated values -> 8 little-endian words of packed codes.
// With z = y + 0 (turns -0 into +0, leaves every other value unchanged) and
// h = m/2, the three comparisons are sign bits of exact sums: [y < -h] is the
// sign of z + h, [y < 0] the sign of z, [y < h] the sign of z - h (a nonzero
// exact sum of two floats never rounds to zero, and x - x = +0).  The code is
// 3 minus their sum, so its high bit is NOT sign(z) and its low bit is
// NOT (sign(z + h) ^ sign(z) ^ sign(z - h)).  The bits are appended most
// significant first with funnel shifts, inverted and byte-reversed at the end.
__device__ __forceinline__ void bucket_pack_thread(const float (&y)[kDim], uint32_t (&w)[kCodeWords]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kDim; ++i) m = fmaxf(m, fabsf(y[i]));
  const float h = 0.5f * m;
#pragma unroll
  for (int i = 0; i < kCodeWords; ++i) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float z = __fadd_rn(y[16 * i + e], 0.0f);
      const uint32_t zb = __float_as_uint(z);
      const uint32_t lo = __float_as_uint(__fadd_rn(z, h)) ^ zb ^ __float_as_uint(__fsub_rn(z, h));
      acc = __funnelshift_l(zb, acc, 1);
      acc = __funnelshift_l(lo, acc, 1);
    }
    w[i] = __byte_perm(~acc, 0u, 0x0123);
  }
}

// ---------------------------------------------------------------- one vector per warp
// Lane L holds elements 4L..4L+3.  Stages h = 1, 2 stay in the lane; stage h >= 4
// pairs lane L with lane L ^ (h / 4): the lane holding x[j] (bit h of j clear)
// computes x[j] + x[j+h], the partner computes x[j] - x[j+h].
// Returns, in every lane, packed code word (lane & 7).
// `raw` holds the lane's four bf16 elements (loaded by encode128_warp_load).
__device__ __forceinline__ uint2 encode128_warp_load(const uint16_t* __restrict__ x, int lane) {
  return *reinterpret_cast<const uint2*>(x + 4 * lane);
}

__device__ __forceinline__ uint32_t encode128_warp_raw(uint2 raw, int lane) {
  float v0 = bf16_lo(raw.x), v1 = bf16_hi(raw.x), v2 = bf16_lo(raw.y), v3 = bf16_hi(raw.y);
  float a, b;
  // h = 1: (0,1) (2,3)
  a = v0; b = v1; v0 = __fadd_rn(a, b); v1 = __fsub_rn(a, b);
  a = v2; b = v3; v2 = __fadd_rn(a, b); v3 = __fsub_rn(a, b);
  // h = 2: (0,2) (1,3)
  a = v0; b = v2; v0 = __fadd_rn(a, b); v2 = __fsub_rn(a, b);
  a = v1; b = v3; v1 = __fadd_rn(a, b); v3 = __fsub_rn(a, b);
#pragma unroll
  for (int lm = 1; lm < 32; lm *= 2) {  // h = 4 * lm
    const bool upper = (lane & lm) != 0;
    const float p0 = __shfl_xor_sync(0xffffffffu, v0, lm);
    const float p1 = __shfl_xor_sync(0xffffffffu, v1, lm);
    const float p2 = __shfl_xor_sync(0xffffffffu, v2, lm);
    const float p3 = __shfl_xor_sync(0xffffffffu, v3, lm);
    v0 = upper ? __fsub_rn(p0, v0) : __fadd_rn(v0, p0);
    v1 = upper ? __fsub_rn(p1, v1) : __fadd_rn(v1, p1);
    v2 = upper ? __fsub_rn(p2, v2) : __fadd_rn(v2, p2);
    v3 = upper ? __fsub_rn(p3, v3) : __fadd_rn(v3, p3);
  }
  const float c = hadamard_norm();
  v0 = __fmul_rn(v0, c); v1 = __fmul_rn(v1, c); v2 = __fmul_rn(v2, c); v3 = __fmul_rn(v3, c);
  float m = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
#pragma unroll
  for (int o = 16; o > 0; o /= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float t0 = -0.5f * m, t2 = 0.5f * m;
  const uint32_t byte = code_of(v0, t0, t2) << 6 | code_of(v1, t0, t2) << 4 |
                        code_of(v2, t0, t2) << 2 | code_of(v3, t0, t2);
  // byte L goes to word L/4 at bit offset 8*(L%4)
  uint32_t w = byte << (8 * (lane & 3));
  w |= __shfl_xor_sync(0xffffffffu, w, 1);
  w |= __shfl_xor_sync(0xffffffffu, w, 2);
  // lane 4i now holds word i; hand word (lane & 7) to every lane
  return __shfl_sync(0xffffffffu, w, 4 * (lane & 7));
}

__device__ __forceinline__ uint32_t encode128_warp(const uint16_t* __restrict__ x, int lane) {
  return encode128_warp_raw(encode128_warp_load(x, lane), lane);
}

}  // namespace adamas
