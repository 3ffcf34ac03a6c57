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

// ---------------------------------------------------------------- one vector per thread, packed pairs
// Packed fp32 pairs (sm_100): every element of the pair is rounded exactly as the
// scalar operation would round it, so a pair instruction is two scalar operations
// for one issue slot.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// P[i] holds the elements (2i, 2i + 1) of one vector.  Stage h = 1 pairs the two
// elements of one register and is done in scalar form as the bf16 words are
// unpacked (rotate_pairs_first); stages h = 2 .. 64 pair register i with register
// i + h/2 (bit h/2 of i clear), both of whose elements are butterfly partners.
template <int HP>
__device__ __forceinline__ void fwht_pair_stage(uint64_t (&P)[kDim / 2]) {
#pragma unroll
  for (int i = 0; i < kDim / 2; i += 2 * HP) {
#pragma unroll
    for (int j = i; j < i + HP; ++j) {
      const uint64_t a = P[j], b = P[j + HP];
      P[j] = f2_add(a, b);
      P[j + HP] = f2_sub(a, b);
    }
  }
}

// Stage h = 1 of the elements held in one packed bf16 word (elements 2i, 2i + 1).
__device__ __forceinline__ uint64_t rotate_pair_first(uint32_t w) {
  const float a = bf16_lo(w), b = bf16_hi(w);
  return f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
}

// Stages h = 2 .. 64, then z = RN(y * C) for every element.  The normalisation is
// one fused multiply-add with +0: its product is exact before the single rounding,
// so z equals RN(y * C) bit for bit, except that a -0 result becomes +0 (which the
// bucketing wants anyway; -0 and +0 compare equal).
__device__ __forceinline__ void rotate_pairs_rest(uint64_t (&P)[kDim / 2]) {
  fwht_pair_stage<1>(P);
  fwht_pair_stage<2>(P);
  fwht_pair_stage<4>(P);
  fwht_pair_stage<8>(P);
  fwht_pair_stage<16>(P);
  fwht_pair_stage<32>(P);
  const float c = hadamard_norm();
  const uint64_t cc = f2_pack(c, c), zero = f2_pack(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < kDim / 2; ++i) P[i] = f2_fma(P[i], cc, zero);
}

// Rotated values (pairs, -0 already +0) -> 8 little-endian words of packed codes.
// With h = m/2 the three comparisons are sign bits of exact sums: [z < -h] is the
// sign of z + h, [z < 0] the sign of z, [z < h] the sign of z - h (a nonzero exact
// sum of two floats never rounds to zero, and x - x = +0).  The code is 3 minus
// their sum, so its high bit is NOT sign(z) and its low bit is
// NOT (sign(z + h) ^ sign(z) ^ sign(z - h)).  The bits are appended most
// significant first with funnel shifts, inverted and byte-reversed at the end.
__device__ __forceinline__ void bucket_pack_pairs(const uint64_t (&P)[kDim / 2], uint32_t (&w)[kCodeWords]) {
  float mm[8];  // eight independent running maxima (short dependency chains)
#pragma unroll
  for (int j = 0; j < 8; ++j) mm[j] = 0.0f;
#pragma unroll
  for (int i = 0; i < kDim / 2; ++i) {
    float a, b;
    f2_unpack(P[i], a, b);
    mm[i & 7] = fmaxf(mm[i & 7], fmaxf(fabsf(a), fabsf(b)));
  }
  const float m = fmaxf(fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])), fmaxf(fmaxf(mm[4], mm[5]), fmaxf(mm[6], mm[7])));
  const float h = 0.5f * m;
  const uint64_t hh = f2_pack(h, h);
  // word i holds the codes of elements 16 i .. 16 i + 15 (pairs 8 i .. 8 i + 7)
  uint32_t acc[kCodeWords];
#pragma unroll
  for (int i = 0; i < kCodeWords; ++i) acc[i] = 0u;
#pragma unroll
  for (int i = 0; i < kCodeWords; ++i) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint64_t z = P[8 * i + q];
      float z0, z1, p0, p1, m0, m1;
      f2_unpack(z, z0, z1);
      f2_unpack(f2_add(z, hh), p0, p1);
      f2_unpack(f2_sub(z, hh), m0, m1);
      const uint32_t zb0 = __float_as_uint(z0), zb1 = __float_as_uint(z1);
      acc[i] = __funnelshift_l(zb0, acc[i], 1);
      acc[i] = __funnelshift_l(__float_as_uint(p0) ^ zb0 ^ __float_as_uint(m0), acc[i], 1);
      acc[i] = __funnelshift_l(zb1, acc[i], 1);
      acc[i] = __funnelshift_l(__float_as_uint(p1) ^ zb1 ^ __float_as_uint(m1), acc[i], 1);
    }
  }
#pragma unroll
  for (int i = 0; i < kCodeWords; ++i) w[i] = __byte_perm(~acc[i], 0u, 0x0123);
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
