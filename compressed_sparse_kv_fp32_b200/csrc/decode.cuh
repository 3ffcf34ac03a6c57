// One ADAMAS decode step as a single cooperative kernel (one block per SM).
//
// Method (ADAMAS long-context sparse attention article, lnwmold.com/news/826806):
// the query is rotated and bucketed like the keys (§2.1, §2.2), every cached
// token is scored by the L1 distance of its 2-bit codes (§2.3), a token budget of
// the best tokens is kept (§5.2) and exact softmax attention runs over their K/V
// rows (the rotation preserves q.k, §2.1, so the exact product uses the original
// vectors).
//
// Work split.  All (b, kv head, token) units of the batch form one range that is
// cut evenly over the S blocks; a block's share may cross kv heads, so it is
// handled as "segments" (the part of one kv head inside the block's share).
//   phase 1  per segment: encode the G query heads of the kv head, stream the
//            segment's packed codes once with 32-byte loads, compute the G
//            distances of every token, keep them in shared memory and build one
//            385-bin histogram per query head; publish the histogram.
//   -- grid-wide wait --
//   phase 2  per segment and query head: sum the head's histograms (one per
//            segment of that head) to get the threshold distance T with
//            count(D < T) < k_eff <= count(D <= T), then place every token with
//            D <= T straight at its final slot of the (D, index)-ordered list:
//            slot = #tokens with smaller D + #tokens with equal D and a lower
//            index (earlier segments from their histograms, earlier warps from a
//            per-warp count, earlier lanes by a warp match); slots >= k_eff are
//            dropped, which keeps ties at T for the lowest indices.  No sort and
//            no candidate list is needed, and the distances never leave the SM.
//   -- grid-wide wait --
//   phase 3  the kept rows of all query heads form a second range, cut evenly
//            over the blocks; every half-warp gathers bf16 K/V rows (16 bytes
//            per lane) and keeps an online-softmax state; each block publishes
//            one partial state per query head it touched, and the last block to
//            finish a query head (atomic ticket, no waiting) merges the partial
//            states into out.
//
// Every grid-wide wait is bounded: after kSpinLimit polls the block sets
// ADAMAS_DEVERR_TIMEOUT in the error word and returns.
#pragma once

#include "common.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kHistStride = 388;      // >= kBins, multiple of 4
constexpr int kPartial = 132;         // m, l, pad, pad, o[128]
constexpr int kRowsPerHalfWarp = 4;   // K/V rows in flight per half-warp
constexpr uint32_t kSpinLimit = 1u << 20;   // about a second of polling

struct DecodeParams {
  const uint16_t* q;
  const uint8_t* codes;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* seq_lens;
  float* out;
  int32_t* idx;
  uint32_t* ctrl;       // [0] wait arrivals, [1] wait generation, [2] error word
  uint32_t* head_done;  // [B*Hq] tickets of phase 3
  uint32_t* hist;       // [(S + B*Hkv) * G][kHistStride]
  float* partial;       // [(S + B*Hq)][kPartial]
  uint16_t* dglobal;    // [S][G][range_cap] when distances do not fit in shared memory
  int B, Hq, Hkv;
  int64_t Nmax;
  int budget;
  int S;
  int64_t range_cap;    // >= units of any block
  int smem_d;           // distances kept in shared memory
};

// Shared-memory carve-up (bytes), shared with the host.
struct DecodeSmem {
  static __host__ __device__ inline size_t meta(int B) { return (size_t)(B + 1) * 16 + (size_t)B * 4; }
  static __host__ __device__ inline size_t qwords(int G) { return (size_t)G * kCodeWords * 4; }
  static __host__ __device__ inline size_t work(int G) {
    const int rows = G > kWarps + 1 ? G : kWarps + 1;
    return (size_t)rows * kHistStride * 4;
  }
  static __host__ __device__ inline size_t dist(int G, int64_t range_cap, bool in_smem) {
    const size_t p3 = (size_t)2 * kWarps * kPartial * 4;
    const size_t dd = in_smem ? (size_t)G * (size_t)((range_cap + 7) / 8 * 8) * 2 : 0;
    return dd > p3 ? dd : p3;
  }
  static __host__ __device__ inline size_t align16(size_t x) { return (x + 15) / 16 * 16; }
  static __host__ __device__ inline size_t total(int B, int G, int64_t range_cap, bool in_smem) {
    return align16(meta(B)) + align16(qwords(G)) + align16(work(G)) + align16(dist(G, range_cap, in_smem));
  }
};

// ------------------------------------------------------------------ block helpers
// Bounded grid-wide wait.  Returns false (in every thread) when it timed out.
__device__ __forceinline__ bool grid_wait(uint32_t* ctrl, int S, int* sm_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint32_t gen = ld_acquire_gpu(ctrl + 1);
    __threadfence();
    const uint32_t arrived = atomicAdd(ctrl, 1u) + 1u;
    if (arrived == (uint32_t)S) {
      atomicExch(ctrl, 0u);
      __threadfence();
      atomicAdd(ctrl + 1, 1u);
    } else {
      uint32_t spins = 0;
      while (ld_acquire_gpu(ctrl + 1) == gen) {
        if (++spins > kSpinLimit) {
          atomicOr(ctrl + 2, kErrTimeout);
          ok = 0;
          break;
        }
        __nanosleep(spins < 64 ? 32 : 256);
      }
    }
    __threadfence();
    *sm_flag = ok;
  }
  __syncthreads();
  return *sm_flag != 0;
}

// Exclusive scan of one int64 per thread over the block; returns the prefix and
// writes the block total to *total.  Uses sm_tmp[kWarps + 1].
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* sm_tmp, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o *= 2) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < kWarps ? sm_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) sm_tmp[lane] = w;  // inclusive warp totals
    if (lane == kWarps - 1) sm_tmp[kWarps] = w;
  }
  __syncthreads();
  const int64_t before = warp > 0 ? sm_tmp[warp - 1] : 0;
  const int64_t res = before + x - v;
  *total = sm_tmp[kWarps];
  __syncthreads();
  return res;
}

// Largest b in [0, B) with off[b] <= x (off nondecreasing, off[0] = 0 <= x).
__device__ __forceinline__ int find_batch(const int64_t* off, int B, int64_t x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Segment {
  int b, kvh, hk;
  int64_t t0;     // first token of the segment within its kv head
  int64_t len;    // tokens in the segment
  int64_t soff;   // offset of the segment within the block's share
  int64_t head_u0;  // first unit of the kv head
};

__device__ __forceinline__ Segment segment_at(int64_t u, int64_t lo, int64_t hi, const int64_t* uoff,
                                              const int32_t* lens, int B, int Hkv) {
  Segment g;
  g.b = find_batch(uoff, B, u);
  const int64_t len = lens[g.b];
  const int64_t rel = u - uoff[g.b];
  g.kvh = (int)(rel / len);
  g.t0 = rel - (int64_t)g.kvh * len;
  g.hk = g.b * Hkv + g.kvh;
  g.head_u0 = uoff[g.b] + (int64_t)g.kvh * len;
  const int64_t end = min(hi, g.head_u0 + len);
  g.len = end - u;
  g.soff = u - lo;
  return g;
}

// ------------------------------------------------------------------ the kernel
template <int G>
__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int sm_flag;
  __shared__ int sm_T;
  __shared__ int sm_last;
  __shared__ int64_t sm_scan[kWarps + 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, S = p.S, B = p.B;

  int64_t* sm_uoff = reinterpret_cast<int64_t*>(smem);                  // [B + 1]
  int64_t* sm_roff = sm_uoff + (B + 1);                                 // [B + 1]
  int32_t* sm_len = reinterpret_cast<int32_t*>(sm_roff + (B + 1));      // [B]
  unsigned char* cur = smem + DecodeSmem::align16(DecodeSmem::meta(B));
  uint32_t* sm_q = reinterpret_cast<uint32_t*>(cur);                    // [G][8]
  cur += DecodeSmem::align16(DecodeSmem::qwords(G));
  uint32_t* sm_work = reinterpret_cast<uint32_t*>(cur);                 // [rows][kHistStride]
  cur += DecodeSmem::align16(DecodeSmem::work(G));
  unsigned char* sm_dist = cur;                                         // distances / phase-3 states

  uint16_t* dbuf = p.smem_d ? reinterpret_cast<uint16_t*>(sm_dist)
                            : p.dglobal + (int64_t)s * G * p.range_cap;
  const int64_t dstride = p.smem_d ? (p.range_cap + 7) / 8 * 8 : p.range_cap;

  // ---- lengths and offsets of the unit range and of the kept-row range
  int64_t uoff_total, roff_total;
  {
    // B <= kMaxBatch = 2 * kThreads: thread i owns batches 2i and 2i+1
    int64_t lu = 0, lr = 0;
    for (int k = 0; k < 2; ++k) {
      const int b = 2 * tid + k;
      if (b < B) {
        int32_t len = p.seq_lens[b];
        if (len < 0 || (int64_t)len > p.Nmax) {
          if (s == 0) atomicOr(p.ctrl + 2, kErrSeqLen);
          len = len < 0 ? 0 : (int32_t)p.Nmax;
        }
        sm_len[b] = len;
        lu += (int64_t)p.Hkv * len;
        lr += (int64_t)p.Hq * min(p.budget, len);
      }
    }
    const int64_t pu = block_exclusive_scan(lu, sm_scan, &uoff_total);
    const int64_t pr = block_exclusive_scan(lr, sm_scan, &roff_total);
    int64_t au = pu, ar = pr;
    for (int k = 0; k < 2; ++k) {
      const int b = 2 * tid + k;
      if (b < B) {
        sm_uoff[b] = au;
        sm_roff[b] = ar;
        au += (int64_t)p.Hkv * sm_len[b];
        ar += (int64_t)p.Hq * min(p.budget, sm_len[b]);
      }
    }
    if (tid == 0) {
      sm_uoff[B] = uoff_total;
      sm_roff[B] = roff_total;
    }
    __syncthreads();
  }
  const int64_t U = uoff_total;
  const int64_t u_lo = U > 0 ? range_begin(s, U, S) : 0;
  const int64_t u_hi = U > 0 ? range_begin(s + 1, U, S) : 0;

  // ================================================================ phase 1
  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    if (warp < G) {
      const int hq = seg.b * p.Hq + seg.kvh * G + warp;
      const uint32_t w = encode128_warp(p.q + (int64_t)hq * kDim, lane);
      if (lane < kCodeWords) sm_q[warp * kCodeWords + lane] = w;
    }
    for (int i = tid; i < G * kHistStride; i += kThreads) sm_work[i] = 0u;
    __syncthreads();

    uint32_t qw[G][kCodeWords];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int w = 0; w < kCodeWords; ++w) qw[g][w] = sm_q[g * kCodeWords + w];

    const uint8_t* crow = p.codes + ((int64_t)seg.hk * p.Nmax + seg.t0) * kCodeBytes;
    constexpr int kUnroll = G <= 2 ? 4 : 2;
    for (int64_t base = 0; base < seg.len; base += (int64_t)kThreads * kUnroll) {
      uint32_t kc[kUnroll][kCodeWords];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int64_t t = base + (int64_t)j * kThreads + tid;
        if (t < seg.len) ld_stream_v8(crow + t * kCodeBytes, kc[j]);
      }
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int64_t t = base + (int64_t)j * kThreads + tid;
        if (t < seg.len) {
          uint32_t e[kCodeWords];
          key_odd_mask(kc[j], e);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int d = l1_distance(kc[j], e, qw[g]);
            dbuf[(int64_t)g * dstride + seg.soff + t] = (uint16_t)d;
            atomicAdd(&sm_work[g * kHistStride + d], 1u);
          }
        }
      }
    }
    __syncthreads();
    for (int i = tid; i < G * kBins; i += kThreads) {
      const int g = i / kBins, d = i - g * kBins;
      p.hist[((int64_t)(s + seg.hk) * G + g) * kHistStride + d] = sm_work[g * kHistStride + d];
    }
    __syncthreads();
    u += seg.len;
  }

  if (!grid_wait(p.ctrl, S, &sm_flag)) return;

  // ================================================================ phase 2
  uint32_t* sm_cnt = sm_work;                          // [kWarps][kHistStride]
  uint32_t* sm_rank = sm_work + kWarps * kHistStride;  // [kHistStride]
  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    const int64_t len_b = sm_len[seg.b];
    const int keff = (int)min((int64_t)p.budget, len_b);
    const int s_first = owner_of(seg.head_u0, U, S);
    const int s_last = owner_of(seg.head_u0 + len_b - 1, U, S);
    for (int g = 0; g < G && keff > 0; ++g) {
      const int64_t hq = (int64_t)seg.b * p.Hq + seg.kvh * G + g;
      int64_t H = 0, P = 0;
      if (tid < kBins) {
        for (int s2 = s_first; s2 <= s_last; ++s2) {
          if (range_begin(s2, U, S) == range_begin(s2 + 1, U, S)) continue;  // block without units
          const uint32_t v = __ldcg(&p.hist[((int64_t)(s2 + seg.hk) * G + g) * kHistStride + tid]);
          H += v;
          if (s2 < s) P += v;
        }
      }
      int64_t tot;
      const int64_t base = block_exclusive_scan(H, sm_scan, &tot);
      if (tid < kBins) {
        if (base < keff && base + H >= keff) sm_T = tid;
        sm_rank[tid] = (uint32_t)(base + P);
      }
      for (int i = tid; i < kWarps * kHistStride; i += kThreads) sm_cnt[i] = 0u;
      __syncthreads();
      const int T = sm_T;
      const uint16_t* dg = dbuf + (int64_t)g * dstride + seg.soff;
      const int64_t chunk = (seg.len + kWarps - 1) / kWarps;
      const int64_t w0 = min(seg.len, (int64_t)warp * chunk), w1 = min(seg.len, w0 + chunk);
      // pass 1: per-warp counts of kept candidates per distance
      for (int64_t i = w0 + lane; i < w1; i += 32) {
        const int d = dg[i];
        if (d <= T) atomicAdd(&sm_cnt[warp * kHistStride + d], 1u);
      }
      __syncthreads();
      if (tid <= T) {
        uint32_t run = 0;
        for (int w = 0; w < kWarps; ++w) {
          const uint32_t c = sm_cnt[w * kHistStride + tid];
          sm_cnt[w * kHistStride + tid] = run;
          run += c;
        }
      }
      __syncthreads();
      // pass 2: in index order, place every candidate at its final slot
      int32_t* idx_h = p.idx + hq * p.budget;
      const uint32_t lt = (1u << lane) - 1u;
      for (int64_t i0 = w0; i0 < w1; i0 += 32) {
        const int64_t i = i0 + lane;
        const int d = i < w1 ? (int)dg[i] : kBins;
        const bool cand = d <= T;
        const uint32_t m = __ballot_sync(0xffffffffu, cand);
        if (m == 0u) continue;
        uint32_t peers = 0;
        if (cand) {
          peers = __match_any_sync(m, d);
          const uint32_t slot = sm_rank[d] + sm_cnt[warp * kHistStride + d] + __popc(peers & lt);
          if (slot < (uint32_t)keff) idx_h[slot] = (int32_t)(seg.t0 + i);
        }
        __syncwarp();
        if (cand && (peers & lt) == 0u) sm_cnt[warp * kHistStride + d] += __popc(peers);
        __syncwarp();
      }
      if (s == s_first)
        for (int r = keff + tid; r < p.budget; r += kThreads) idx_h[r] = -1;
      __syncthreads();
    }
    u += seg.len;
  }
  // query heads that keep no token: out = 0, idx = -1
  for (int64_t hq = s; hq < (int64_t)B * p.Hq; hq += S) {
    const int b = (int)(hq / p.Hq);
    if (min(p.budget, sm_len[b]) > 0) continue;
    for (int i = tid; i < kDim; i += kThreads) p.out[hq * kDim + i] = 0.0f;
    for (int r = tid; r < p.budget; r += kThreads) p.idx[hq * p.budget + r] = -1;
  }

  if (!grid_wait(p.ctrl, S, &sm_flag)) return;

  // ================================================================ phase 3
  const int64_t R = roff_total;
  const int64_t r_lo = R > 0 ? range_begin(s, R, S) : 0;
  const int64_t r_hi = R > 0 ? range_begin(s + 1, R, S) : 0;
  float* sm_state = reinterpret_cast<float*>(sm_dist);   // [2*kWarps][kPartial]
  const int hw = tid >> 4, hl = tid & 15;
  const float kScoreScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e)/sqrt(128)
  for (int64_t r = r_lo; r < r_hi;) {
    const int b = find_batch(sm_roff, B, r);
    const int keff = min(p.budget, sm_len[b]);
    const int64_t rel = r - sm_roff[b];
    const int h = (int)(rel / keff);
    const int64_t j0 = rel - (int64_t)h * keff;
    const int64_t head_r0 = sm_roff[b] + (int64_t)h * keff;
    const int64_t slen = min(r_hi, head_r0 + keff) - r;
    const int64_t hq = (int64_t)b * p.Hq + h;
    const int kvh = h / G;
    const int64_t len_b = sm_len[b];
    const int64_t kv_base = ((int64_t)b * p.Hkv + kvh) * p.Nmax;

    float qf[8];
    {
      const uint4 qr = *reinterpret_cast<const uint4*>(p.q + hq * kDim + 8 * hl);
      qf[0] = bf16_lo(qr.x) * kScoreScale; qf[1] = bf16_hi(qr.x) * kScoreScale;
      qf[2] = bf16_lo(qr.y) * kScoreScale; qf[3] = bf16_hi(qr.y) * kScoreScale;
      qf[4] = bf16_lo(qr.z) * kScoreScale; qf[5] = bf16_hi(qr.z) * kScoreScale;
      qf[6] = bf16_lo(qr.w) * kScoreScale; qf[7] = bf16_hi(qr.w) * kScoreScale;
    }
    float m_run = -INFINITY, l_run = 0.0f, o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = 0.0f;

    const int32_t* idx_h = p.idx + hq * p.budget + j0;
    // The trip count depends on the warp only, so both half-warps always reach
    // the full-warp shuffles below together.
    for (int64_t jb = 2 * warp; jb < slen; jb += 2 * kWarps * kRowsPerHalfWarp) {
      int32_t t[kRowsPerHalfWarp];
      uint4 kr[kRowsPerHalfWarp], vr[kRowsPerHalfWarp];
#pragma unroll
      for (int u2 = 0; u2 < kRowsPerHalfWarp; ++u2) {
        const int64_t jj = jb + (hw & 1) + (int64_t)u2 * 2 * kWarps;
        t[u2] = jj < slen ? __ldcg(idx_h + jj) : -1;
        if (t[u2] >= len_b) t[u2] = -1;  // never read outside the sequence
      }
#pragma unroll
      for (int u2 = 0; u2 < kRowsPerHalfWarp; ++u2) {
        if (t[u2] >= 0) {
          const int64_t off = (kv_base + t[u2]) * kDim + 8 * hl;
          kr[u2] = __ldg(reinterpret_cast<const uint4*>(p.K + off));
          vr[u2] = __ldg(reinterpret_cast<const uint4*>(p.V + off));
        }
      }
#pragma unroll
      for (int u2 = 0; u2 < kRowsPerHalfWarp; ++u2) {
        const bool valid = t[u2] >= 0;  // uniform across the half-warp
        float sc = 0.0f;
        if (valid)
          sc = qf[0] * bf16_lo(kr[u2].x) + qf[1] * bf16_hi(kr[u2].x) + qf[2] * bf16_lo(kr[u2].y) +
               qf[3] * bf16_hi(kr[u2].y) + qf[4] * bf16_lo(kr[u2].z) + qf[5] * bf16_hi(kr[u2].z) +
               qf[6] * bf16_lo(kr[u2].w) + qf[7] * bf16_hi(kr[u2].w);
        sc += __shfl_xor_sync(0xffffffffu, sc, 8);
        sc += __shfl_xor_sync(0xffffffffu, sc, 4);
        sc += __shfl_xor_sync(0xffffffffu, sc, 2);
        sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        if (!valid) continue;
        const float m_new = fmaxf(m_run, sc);
        const float corr = exp2f(m_run - m_new);
        const float pr = exp2f(sc - m_new);
        l_run = l_run * corr + pr;
        const float vv[8] = {bf16_lo(vr[u2].x), bf16_hi(vr[u2].x), bf16_lo(vr[u2].y), bf16_hi(vr[u2].y),
                             bf16_lo(vr[u2].z), bf16_hi(vr[u2].z), bf16_lo(vr[u2].w), bf16_hi(vr[u2].w)};
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = o[e] * corr + pr * vv[e];
        m_run = m_new;
      }
    }
    // half-warp states -> block partial
    float* st = sm_state + hw * kPartial;
    if (hl == 0) { st[0] = m_run; st[1] = l_run; }
#pragma unroll
    for (int e = 0; e < 8; ++e) st[4 + 8 * hl + e] = o[e];
    __syncthreads();
    const int slot = (int)(s + hq);
    float* part = p.partial + (int64_t)slot * kPartial;
    if (tid < kDim) {
      float M = -INFINITY;
      for (int k = 0; k < 2 * kWarps; ++k) M = fmaxf(M, sm_state[k * kPartial]);
      float L = 0.0f, O = 0.0f;
      for (int k = 0; k < 2 * kWarps; ++k) {
        const float* sk = sm_state + k * kPartial;
        const float wgt = exp2f(sk[0] - M);  // 0 for a half-warp without rows
        L += sk[1] * wgt;
        O += sk[4 + tid] * wgt;
      }
      part[4 + tid] = O;
      if (tid == 0) { part[0] = M; part[1] = L; }
    }
    __threadfence();
    __syncthreads();
    const int sf = owner_of(head_r0, R, S), sl = owner_of(head_r0 + keff - 1, R, S);
    if (tid == 0) {
      uint32_t slices = 0;  // blocks of [sf, sl] that hold rows of this head
      for (int s2 = sf; s2 <= sl; ++s2) slices += range_begin(s2, R, S) != range_begin(s2 + 1, R, S);
      const uint32_t prev = atomicAdd(&p.head_done[hq], 1u);
      sm_last = prev + 1u == slices;
    }
    __syncthreads();
    if (sm_last) {
      __threadfence();
      if (tid < kDim) {
        float M = -INFINITY;
        for (int s2 = sf; s2 <= sl; ++s2)
          if (range_begin(s2, R, S) != range_begin(s2 + 1, R, S))
            M = fmaxf(M, __ldcg(p.partial + (int64_t)(s2 + hq) * kPartial));
        float L = 0.0f, O = 0.0f;
        for (int s2 = sf; s2 <= sl; ++s2) {
          if (range_begin(s2, R, S) == range_begin(s2 + 1, R, S)) continue;
          const float* ps = p.partial + (int64_t)(s2 + hq) * kPartial;
          const float wgt = exp2f(__ldcg(ps) - M);
          L += __ldcg(ps + 1) * wgt;
          O += __ldcg(ps + 4 + tid) * wgt;
        }
        p.out[hq * kDim + tid] = O / L;
      }
      if (tid == 0) p.head_done[hq] = 0u;
    }
    __syncthreads();
    r += slen;
  }
}

}  // namespace adamas
