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
// cut evenly over Sr <= S blocks (when every sequence has the same length and
// there are no more kv heads than blocks, Sr is a multiple of the number of kv
// heads so that no block straddles two heads); a block's share is handled as
// "segments" (the part of one kv head inside the block's share).
//   phase 1  per segment: encode the G query heads of the kv head, stream the
//            packed code rows with 32-byte loads (eight rows in flight per thread,
//            256 KiB per block), keep the G distances of
//            every token in shared memory and add them to one 385-bin histogram
//            per query head; publish the histograms.
//   -- grid-wide wait --
//   phase 2  per segment and query head: sum the head's histograms (one per
//            segment of that head, loaded together) to get the threshold T with
//            count(D < T) < k_eff <= count(D <= T).  Pass 1: each warp scans its
//            slice of the distances eight at a time and counts the tokens with
//            D <= T per distance; prefix sums over warps then give every warp
//            the number of tokens it keeps and where its kept tokens go in a
//            block list.  Pass 2: each warp scans again in index order and puts
//            every candidate straight at its final slot of the (D, index)-ordered
//            output: slot = #tokens with smaller D + #tokens with equal D and a
//            lower index (earlier segments from their histograms, earlier warps
//            from the per-warp counts, earlier lanes by a warp match).  Slots
//            >= k_eff are dropped, which keeps ties at T for the lowest indices.
//            The block then gathers the K and V rows of its kept tokens (16-byte
//            cp.async copies, double-buffered), every half-warp keeps an
//            online-softmax state, and the block publishes one partial state for
//            the query head; the last block to publish for a query head (atomic
//            ticket, no waiting) merges the partials into out.
//
// The grid-wide wait is bounded: it gives up after kSpinLimit polls and sets
// ADAMAS_DEVERR_TIMEOUT.
#pragma once

#include "common.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

constexpr int kThreads = 512;
constexpr int kBlocksPerSM = 1;
constexpr int kWarps = kThreads / 32;
constexpr int kBatchPerThread = kMaxBatch / kThreads;
constexpr int kBinsPerThread = (kBins + kThreads - 1) / kThreads;
constexpr int kHistStride = 388;                     // >= kBins, multiple of 4
constexpr int kPartial = 132;                        // m, l, pad, pad, o[128]
constexpr uint32_t kRowBytes = 2 * kDim * 2;         // one K row + one V row (bf16)
constexpr int kScratch = 256;                        // candidate entries per warp per 256-token group
constexpr int kMaxKept = 1024;                       // kept tokens listed per sweep
constexpr int kMaxRowsStaged = 256;
constexpr int kMinRowsStaged = 32;
constexpr int kMaxBlocks = 1024;
constexpr uint32_t kSpinLimit = 1u << 20;            // grid-wide wait polls (about a second)

struct DecodeParams {
  const uint16_t* q;
  const uint8_t* codes;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* seq_lens;
  float* out;
  int32_t* idx;
  uint32_t* ctrl;       // [0..1] grid-wait word (generation << 32 | arrivals), [2] error word
  uint32_t* head_done;  // [B*Hq] merge tickets
  uint32_t* hist;       // [(S + B*Hkv) * G][kHistStride]
  float* partial;       // [(S + B*Hkv) * G][kPartial]
  uint16_t* dglobal;    // [S][G][dstride] when distances do not fit in shared memory
  int B, Hq, Hkv;
  int64_t Nmax;
  int budget;
  int S;
  int64_t range_cap;    // >= units of any block
  int smem_d;           // distances kept in shared memory
  int row_cap;          // K/V rows of the dedicated gather staging (even; 0 with stage_in_d)
  int stage_in_d;       // stage gathered rows over the finished distance row instead
};

// Shared-memory carve-up (bytes), shared with the host.
struct DecodeSmem {
  static __host__ __device__ inline size_t align128(size_t x) { return (x + 127) / 128 * 128; }
  static __host__ __device__ inline size_t meta(int B) { return (size_t)(B + 1) * 8 + (size_t)B * 4; }
  static __host__ __device__ inline size_t qwords(int G) { return (size_t)G * kCodeWords * 4; }
  // histograms (phase 1); per-warp counts + rank bases, then the half-warp
  // softmax states (phase 2)
  static __host__ __device__ inline size_t work(int G) {
    const int rows = G > kWarps + 1 ? G : kWarps + 1;
    return (size_t)rows * kHistStride * 4;
  }
  static __host__ __device__ inline size_t scratch() { return (size_t)kWarps * kScratch * 4; }
  static __host__ __device__ inline size_t kept() { return (size_t)kMaxKept * 4; }
  static __host__ __device__ inline int64_t dstride(int64_t range_cap) { return (range_cap + 63) / 64 * 64; }
  static __host__ __device__ inline size_t dist(int G, int64_t range_cap, bool in_smem) {
    return in_smem ? (size_t)G * (size_t)dstride(range_cap) * 2 : 0;
  }
  static __host__ __device__ inline size_t fixed(int B, int G) {
    return align128(meta(B)) + align128(qwords(G)) + align128(work(G)) + align128(scratch()) + align128(kept());
  }
  static __host__ __device__ inline size_t total(int B, int G, int64_t range_cap, bool in_smem, int row_cap) {
    return fixed(B, G) + align128(dist(G, range_cap, in_smem)) + (size_t)row_cap * kRowBytes;
  }
};

// ------------------------------------------------------------------ block helpers
// Bounded grid-wide wait on the word ctrl[0..1] = generation << 32 | arrivals.
// `gen` is the generation current when this wait began (thread 0 only).  Each
// block arrives with one acquire-release add; the last one clears the arrivals
// and advances the generation with one release add, which the others observe
// with acquire loads.  Returns false (in every thread) when the wait timed out.
__device__ __forceinline__ bool grid_wait(uint32_t* ctrl, int S, uint32_t gen, int* sm_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    unsigned long long* word = reinterpret_cast<unsigned long long*>(ctrl);
    const unsigned long long old = atom_add_acqrel_gpu64(word, 1ull);
    if ((uint32_t)old == (uint32_t)(S - 1)) {
      red_add_release_gpu64(word, (1ull << 32) - (unsigned long long)S);
    } else {
      uint32_t spins = 0;
      while ((uint32_t)(ld_acquire_gpu64(word) >> 32) == gen) {
        if (++spins > kSpinLimit) {
          atomicOr(ctrl + 2, kErrTimeout);
          ok = 0;
          break;
        }
        if (spins > 64) __nanosleep(32);
      }
    }
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

// Warp 0 lists, in order, the blocks of [first, last] whose share of a range of
// `total` units is not empty.  Returns the count (valid in warp 0).
__device__ __forceinline__ int list_blocks(int first, int last, int64_t total, int S, int* list) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int base = first; base <= last; base += 32) {
    const int s2 = base + lane;
    const bool ok = s2 <= last && range_begin(s2, total, S) != range_begin(s2 + 1, total, S);
    const uint32_t m = __ballot_sync(0xffffffffu, ok);
    if (ok) list[n + __popc(m & ((1u << lane) - 1u))] = s2;
    n += __popc(m);
  }
  return n;
}

struct Segment {
  int b, kvh, hk;
  int64_t t0;       // first token of the segment within its kv head
  int64_t len;      // tokens in the segment
  int64_t soff;     // offset of the segment within the block's share
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

// ------------------------------------------------------------------ phase-1 helpers
// Rows base + j*kThreads + tid (j < U) of a segment's code rows, 32 bytes each.
template <int U>
__device__ __forceinline__ void load_rows(uint32_t (&dst)[U][kCodeWords], const uint8_t* crow, int base,
                                          int seg_len, int tid) {
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int t = base + j * kThreads + tid;
    if (t < seg_len) ld_stream_v8(crow + (size_t)t * kCodeBytes, dst[j]);
  }
}

// Distances of those rows to the G query codes: stored at dseg[g*dstride + t]
// and counted in the per-head histograms.
template <int G, int U>
__device__ __forceinline__ void score_rows(const uint32_t (&src)[U][kCodeWords], const uint32_t (&qw)[G][kCodeWords],
                                           int base, int seg_len, int tid, uint16_t* dseg, int64_t dstride,
                                           uint32_t* hist) {
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int t = base + j * kThreads + tid;
    if (t < seg_len) {
      uint32_t e[kCodeWords];
      key_odd_mask(src[j], e);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int d = l1_distance(src[j], e, qw[g]);
        dseg[(size_t)g * dstride + t] = (uint16_t)d;
        atomicAdd(&hist[g * kHistStride + d], 1u);
      }
    }
  }
}

// Distances of eight consecutive positions 8*grp .. 8*grp+7 (0xFFFF where grp is
// past the warp's slice).
__device__ __forceinline__ void load_dist8(const uint16_t* drow, int grp, bool in, uint32_t (&d)[8]) {
  uint4 v = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
  if (in) v = *reinterpret_cast<const uint4*>(drow + (size_t)grp * 8);
  d[0] = v.x & 0xFFFFu; d[1] = v.x >> 16; d[2] = v.y & 0xFFFFu; d[3] = v.y >> 16;
  d[4] = v.z & 0xFFFFu; d[5] = v.z >> 16; d[6] = v.w & 0xFFFFu; d[7] = v.w >> 16;
}

// ------------------------------------------------------------------ the kernel
// SMEM_D: the distances of the block's share live in shared memory (else in the
// workspace).
template <int G, bool SMEM_D>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int sm_flag;
  __shared__ int sm_T;
  __shared__ int sm_last;
  __shared__ int sm_nlist;
  __shared__ int sm_kept_total;
  __shared__ int sm_wlt[kWarps];    // per warp: candidates with D < T
  __shared__ int sm_weq[kWarps];    // per warp: candidates with D == T
  __shared__ int sm_wkept[kWarps];  // per warp: first position of its kept tokens in the block list
  __shared__ int64_t sm_scan[kWarps + 1];
  __shared__ int sm_list[kMaxBlocks];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, S = p.S, B = p.B;
  const uint32_t lt = (1u << lane) - 1u;

  int64_t* sm_uoff = reinterpret_cast<int64_t*>(smem);                  // [B + 1]
  int32_t* sm_len = reinterpret_cast<int32_t*>(sm_uoff + (B + 1));      // [B]
  unsigned char* cur = smem + DecodeSmem::align128(DecodeSmem::meta(B));
  uint32_t* sm_q = reinterpret_cast<uint32_t*>(cur);                    // [G][8]
  cur += DecodeSmem::align128(DecodeSmem::qwords(G));
  uint32_t* sm_work = reinterpret_cast<uint32_t*>(cur);                 // [rows][kHistStride]
  cur += DecodeSmem::align128(DecodeSmem::work(G));
  uint32_t* sm_scratch = reinterpret_cast<uint32_t*>(cur);              // [kWarps][kScratch]
  cur += DecodeSmem::align128(DecodeSmem::scratch());
  int32_t* sm_kept = reinterpret_cast<int32_t*>(cur);                   // [kMaxKept]
  cur += DecodeSmem::align128(DecodeSmem::kept());
  const int64_t dstride = DecodeSmem::dstride(p.range_cap);
  uint16_t* dbuf;
  if constexpr (SMEM_D) {
    dbuf = reinterpret_cast<uint16_t*>(cur);                            // [G][dstride]
    cur += DecodeSmem::align128(DecodeSmem::dist(G, p.range_cap, true));
  } else {
    dbuf = p.dglobal + (int64_t)s * G * dstride;
  }
  unsigned char* sm_rows = cur;                                         // [row_cap][512]

  uint32_t gen0 = 0;
  if (tid == 0) gen0 = (uint32_t)(ld_relaxed_gpu64(reinterpret_cast<const unsigned long long*>(p.ctrl)) >> 32);

  // ---- lengths and unit offsets per sequence
  int64_t U;
  int uniform;
  {
    // B <= kMaxBatch: thread i owns batches kBatchPerThread*i + k
    int64_t lu = 0;
    for (int k = 0; k < kBatchPerThread; ++k) {
      const int b = kBatchPerThread * tid + k;
      if (b < B) {
        int32_t len = p.seq_lens[b];
        if (len < 0 || (int64_t)len > p.Nmax) {
          if (s == 0) atomicOr(p.ctrl + 2, kErrSeqLen);
          len = len < 0 ? 0 : (int32_t)p.Nmax;
        }
        sm_len[b] = len;
        lu += (int64_t)p.Hkv * len;
      }
    }
    const int64_t pu = block_exclusive_scan(lu, sm_scan, &U);
    int64_t au = pu;
    int same = 1;
    for (int k = 0; k < kBatchPerThread; ++k) {
      const int b = kBatchPerThread * tid + k;
      if (b < B) {
        sm_uoff[b] = au;
        au += (int64_t)p.Hkv * sm_len[b];
        same &= sm_len[b] == sm_len[0];
      }
    }
    if (tid == 0) sm_uoff[B] = U;
    uniform = __syncthreads_and(same);
  }
  // Blocks the units are split over: a multiple of the kv-head count when every
  // sequence has the same length, so that no block straddles two kv heads.
  const int heads = B * p.Hkv;
  const int Sr = (uniform && heads <= S && U > 0) ? (S / heads) * heads : S;
  const int64_t u_lo = (U > 0 && s < Sr) ? range_begin(s, U, Sr) : 0;
  int64_t u_hi = (U > 0 && s < Sr) ? range_begin(s + 1, U, Sr) : 0;
  if (u_hi - u_lo > p.range_cap) {  // never with the host's sizing; refuse rather than overrun
    atomicOr(p.ctrl + 2, kErrInternal);
    u_hi = u_lo;
  }

  // ================================================================ phase 1
  constexpr int kU = G <= 2 ? 8 : 4;  // code rows in flight per thread
  constexpr int kPerIt = kThreads * kU;
  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    const uint8_t* crow = p.codes + ((int64_t)seg.hk * p.Nmax + seg.t0) * kCodeBytes;
    const int seg_len = (int)seg.len;  // < 2^23 (checked by the host)
    uint16_t* dseg = dbuf + seg.soff;
    // the query rows go first: loads issued after 128 KiB of code rows would
    // queue behind them
    uint2 qraw = make_uint2(0u, 0u);
    if (warp < G) qraw = encode128_warp_load(p.q + ((int64_t)seg.b * p.Hq + seg.kvh * G + warp) * kDim, lane);
    uint32_t kc[kU][kCodeWords];
    load_rows<kU>(kc, crow, 0, seg_len, tid);  // in flight while the query is encoded
    if (warp < G) {
      const uint32_t w = encode128_warp_raw(qraw, lane);
      if (lane < kCodeWords) sm_q[warp * kCodeWords + lane] = w;
    }
    for (int i = tid; i < G * kHistStride; i += kThreads) sm_work[i] = 0u;
    __syncthreads();
    uint32_t qw[G][kCodeWords];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int w = 0; w < kCodeWords; ++w) qw[g][w] = sm_q[g * kCodeWords + w];

    for (int base = 0; base < seg_len; base += kPerIt) {
      if (base > 0) load_rows<kU>(kc, crow, base, seg_len, tid);
      score_rows<G, kU>(kc, qw, base, seg_len, tid, dseg, dstride, sm_work);
    }
    __syncthreads();
    for (int i = tid; i < G * kBins; i += kThreads) {
      const int g = i / kBins, d = i - g * kBins;
      p.hist[((int64_t)(s + seg.hk) * G + g) * kHistStride + d] = sm_work[g * kHistStride + d];
    }
    __syncthreads();
    u += seg.len;
  }

  if (!grid_wait(p.ctrl, S, gen0, &sm_flag)) return;

  // ================================================================ phase 2
  uint32_t* sm_cnt = sm_work;                          // [kWarps][kHistStride]
  uint32_t* sm_rank = sm_work + kWarps * kHistStride;  // [kHistStride]
  float* sm_state = reinterpret_cast<float*>(sm_work); // [2*kWarps][kPartial], after the gather
  uint32_t* scr = sm_scratch + warp * kScratch;

  const int hw = tid >> 4, hl = tid & 15;
  const float kScoreScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e)/sqrt(128)

  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    const int64_t len_b = sm_len[seg.b];
    const int keff = (int)min((int64_t)p.budget, len_b);
    const int seg_len = (int)seg.len, soff = (int)seg.soff;
    if (keff > 0) {
      if (warp == 0) {
        const int n = list_blocks(owner_of(seg.head_u0, U, Sr), owner_of(seg.head_u0 + len_b - 1, U, Sr), U, Sr,
                                  sm_list);
        if (lane == 0) sm_nlist = n;
      }
      __syncthreads();
      const int nlist = sm_nlist;
      const bool first_segment = sm_list[0] == s;
      const int64_t kv_base = (int64_t)seg.hk * p.Nmax;
      // warp slices over 8-position groups of the segment's distances
      const int a0 = soff, a1 = soff + seg_len;
      const int grp0 = a0 >> 3, ngrp = ((a1 + 7) >> 3) - grp0;
      const int gpw = (ngrp + kWarps - 1) / kWarps;
      const int wg0 = grp0 + min(ngrp, warp * gpw), wg1 = grp0 + min(ngrp, (warp + 1) * gpw);
      for (int g = 0; g < G; ++g) {
        const int64_t hq = (int64_t)seg.b * p.Hq + seg.kvh * G + g;
        int32_t* idx_h = p.idx + hq * p.budget;
        const uint16_t* drow = dbuf + (size_t)g * dstride;
        // gathered rows go over this segment's slice of the distance row just
        // selected (free once its pass 2 is done; one sweep only) when it holds
        // 64 rows or more, else to the dedicated area
        unsigned char* stage = sm_rows;
        int stage_cap = p.row_cap;
        if (SMEM_D && p.stage_in_d) {
          const size_t b0 = ((size_t)g * dstride + soff) * 2, b1 = b0 + (size_t)seg_len * 2;
          const size_t a = (b0 + 127) / 128 * 128;
          const int cap = b1 > a ? (int)min((size_t)kMaxRowsStaged, (b1 - a) / kRowBytes) & ~1 : 0;
          if (cap >= 64) {
            stage = reinterpret_cast<unsigned char*>(dbuf) + a;
            stage_cap = cap;
          }
        }
        const int half = stage_cap / 2;
        // ---- threshold and rank bases from the head's histograms; thread i owns
        // the distances kBinsPerThread*i + k
        int64_t H[kBinsPerThread], P[kBinsPerThread];
#pragma unroll
        for (int k = 0; k < kBinsPerThread; ++k) {
          H[k] = 0;
          P[k] = 0;
        }
        for (int k0 = 0; k0 < nlist; k0 += 8) {
          uint32_t v[8][kBinsPerThread];
#pragma unroll
          for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int k = 0; k < kBinsPerThread; ++k) {
              const int d = kBinsPerThread * tid + k;
              v[j][k] = (k0 + j < nlist && d < kBins)
                            ? __ldcg(&p.hist[((int64_t)(sm_list[k0 + j] + seg.hk) * G + g) * kHistStride + d])
                            : 0u;
            }
#pragma unroll
          for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int k = 0; k < kBinsPerThread; ++k) {
              H[k] += v[j][k];
              if (k0 + j < nlist && sm_list[k0 + j] < s) P[k] += v[j][k];
            }
        }
        int64_t hsum = 0;
#pragma unroll
        for (int k = 0; k < kBinsPerThread; ++k) hsum += H[k];
        int64_t tot;
        int64_t base = block_exclusive_scan(hsum, sm_scan, &tot);
#pragma unroll
        for (int k = 0; k < kBinsPerThread; ++k) {
          const int d = kBinsPerThread * tid + k;
          if (d < kBins) {
            if (base < keff && base + H[k] >= keff) sm_T = d;
            sm_rank[d] = (uint32_t)(base + P[k]);
          }
          base += H[k];
        }
        __syncthreads();
        const uint32_t T = (uint32_t)sm_T;

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

        // sweeps of at most kMaxKept kept tokens (one sweep when budget <= kMaxKept)
        for (int c0 = 0;; c0 += kMaxKept) {
          for (int i = tid; i < kWarps * kHistStride; i += kThreads) sm_cnt[i] = 0u;
          __syncthreads();
          // ---- pass 1: per-warp counts of the candidates (D <= T) per distance
          int nlt = 0, neq = 0;
          for (int gb = wg0; gb < wg1; gb += 32) {
            const int grp = gb + lane;
            uint32_t dv[8];
            load_dist8(drow, grp, grp < wg1, dv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int pos = grp * 8 + e;
              if (dv[e] <= T && pos >= a0 && pos < a1) {
                atomicAdd(&sm_cnt[warp * kHistStride + dv[e]], 1u);
                nlt += dv[e] < T;
                neq += dv[e] == T;
              }
            }
          }
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 /= 2) {
            nlt += __shfl_xor_sync(0xffffffffu, nlt, o2);
            neq += __shfl_xor_sync(0xffffffffu, neq, o2);
          }
          if (lane == 0) {
            sm_wlt[warp] = nlt;
            sm_weq[warp] = neq;
          }
          __syncthreads();
          for (int d = tid; d <= (int)T; d += kThreads) {  // exclusive prefix over the warps, per distance
            uint32_t run = 0;
            for (int w = 0; w < kWarps; ++w) {
              const uint32_t c = sm_cnt[w * kHistStride + d];
              sm_cnt[w * kHistStride + d] = run;
              run += c;
            }
          }
          if (tid == 0) {  // kept tokens per warp: every D < T, and the ties at T within the quota
            const int tie0 = (int)sm_rank[T];
            int ties_before = 0, kept_before = 0;
            for (int w = 0; w < kWarps; ++w) {
              const int ties = min(max(keff - (tie0 + ties_before), 0), sm_weq[w]);
              sm_wkept[w] = kept_before;
              kept_before += sm_wlt[w] + ties;
              ties_before += sm_weq[w];
            }
            sm_kept_total = kept_before;
          }
          __syncthreads();
          const int kept_total = sm_kept_total;
          // ---- pass 2: in index order, every candidate to its final slot
          int kept_at = sm_wkept[warp];
          for (int gb = wg0; gb < wg1; gb += 32) {
            const int grp = gb + lane;
            uint32_t dv[8];
            load_dist8(drow, grp, grp < wg1, dv);
            uint32_t mask = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int pos = grp * 8 + e;
              if (dv[e] <= T && pos >= a0 && pos < a1) mask |= 1u << e;
            }
            const int c = __popc(mask);
            if (__ballot_sync(0xffffffffu, c != 0) == 0u) continue;
            int incl = c;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 *= 2) {
              const int y = __shfl_up_sync(0xffffffffu, incl, o2);
              if (lane >= o2) incl += y;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            int at = incl - c;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (mask & (1u << e)) scr[at++] = (uint32_t)(grp * 8 + e - soff) << 9 | dv[e];
            __syncwarp();
            for (int k0 = 0; k0 < total; k0 += 32) {
              const int k = k0 + lane;
              const bool valid = k < total;
              const uint32_t ent = valid ? scr[k] : 0u;
              const uint32_t d = ent & 511u;
              const uint32_t m = __ballot_sync(0xffffffffu, valid);
              uint32_t peers = 0;
              bool kept = false;
              if (valid) {
                peers = __match_any_sync(m, d);
                const uint32_t slot = sm_rank[d] + sm_cnt[warp * kHistStride + d] + __popc(peers & lt);
                if (slot < (uint32_t)keff) {
                  kept = true;
                  if (c0 == 0) idx_h[slot] = (int32_t)(seg.t0 + (int64_t)(ent >> 9));
                }
              }
              const uint32_t kb = __ballot_sync(0xffffffffu, kept);
              const int pos_k = kept_at + __popc(kb & lt);
              if (kept && pos_k >= c0 && pos_k < c0 + kMaxKept) sm_kept[pos_k - c0] = (int32_t)(ent >> 9);
              kept_at += __popc(kb);
              __syncwarp();
              if (valid && (peers & lt) == 0u) sm_cnt[warp * kHistStride + d] += __popc(peers);
              __syncwarp();
            }
          }
          __syncthreads();
          // ---- gather the listed kept rows, double-buffered halves of the staging area
          const int n_list = max(0, min(kMaxKept, kept_total - c0));
          const int nch = (n_list + half - 1) / half;
          auto issue = [&](int ch) {
            const int r0 = ch * half, n = min(half, n_list - r0);
            unsigned char* buf = stage + (size_t)(ch & 1) * half * kRowBytes;
            for (int c = tid; c < n * 32; c += kThreads) {
              const int row = c >> 5, piece = c & 31;
              const int64_t t = seg.t0 + sm_kept[r0 + row];
              const uint16_t* srcp = (piece < 16 ? p.K : p.V) + (kv_base + t) * kDim + (piece & 15) * 8;
              cp_async16(buf + (size_t)row * kRowBytes + piece * 16, srcp);
            }
            cp_async_commit();
          };
          if (nch > 0) issue(0);
          for (int ch = 0; ch < nch; ++ch) {
            if (ch + 1 < nch) {
              issue(ch + 1);
              cp_async_wait<1>();
            } else {
              cp_async_wait<0>();
            }
            __syncthreads();
            const int n = min(half, n_list - ch * half);
            const unsigned char* buf = stage + (size_t)(ch & 1) * half * kRowBytes;
            // The trip count depends on the warp only, so both half-warps always
            // reach the full-warp shuffles below together.
            for (int rb = 2 * warp; rb < n; rb += 2 * kWarps) {
              const int row = rb + (hw & 1);
              const bool valid = row < n;
              float sc = 0.0f;
              uint4 vr = make_uint4(0, 0, 0, 0);
              if (valid) {
                const uint4 kr = *reinterpret_cast<const uint4*>(buf + (size_t)row * kRowBytes + 16 * hl);
                vr = *reinterpret_cast<const uint4*>(buf + (size_t)row * kRowBytes + kDim * 2 + 16 * hl);
                sc = qf[0] * bf16_lo(kr.x) + qf[1] * bf16_hi(kr.x) + qf[2] * bf16_lo(kr.y) + qf[3] * bf16_hi(kr.y) +
                     qf[4] * bf16_lo(kr.z) + qf[5] * bf16_hi(kr.z) + qf[6] * bf16_lo(kr.w) + qf[7] * bf16_hi(kr.w);
              }
              sc += __shfl_xor_sync(0xffffffffu, sc, 8);
              sc += __shfl_xor_sync(0xffffffffu, sc, 4);
              sc += __shfl_xor_sync(0xffffffffu, sc, 2);
              sc += __shfl_xor_sync(0xffffffffu, sc, 1);
              if (!valid) continue;
              const float m_new = fmaxf(m_run, sc);
              const float corr = exp2f(m_run - m_new);
              const float pr = exp2f(sc - m_new);
              l_run = l_run * corr + pr;
              const float vv[8] = {bf16_lo(vr.x), bf16_hi(vr.x), bf16_lo(vr.y), bf16_hi(vr.y),
                                   bf16_lo(vr.z), bf16_hi(vr.z), bf16_lo(vr.w), bf16_hi(vr.w)};
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = o[e] * corr + pr * vv[e];
              m_run = m_new;
            }
            __syncthreads();
          }
          if (c0 + kMaxKept >= kept_total) break;
        }
        if (first_segment)
          for (int r = keff + tid; r < p.budget; r += kThreads) idx_h[r] = -1;
        // ---- half-warp states -> this block's partial state for the query head
        {
          float* st = sm_state + hw * kPartial;
          if (hl == 0) { st[0] = m_run; st[1] = l_run; }
#pragma unroll
          for (int e = 0; e < 8; ++e) st[4 + 8 * hl + e] = o[e];
        }
        __syncthreads();
        float* part = p.partial + ((int64_t)(s + seg.hk) * G + g) * kPartial;
        if (tid < kDim) {
          float M = -INFINITY;
          for (int k = 0; k < 2 * kWarps; ++k) M = fmaxf(M, sm_state[k * kPartial]);
          float L = 0.0f, O = 0.0f;
          if (M != -INFINITY) {
            for (int k = 0; k < 2 * kWarps; ++k) {
              const float* sk = sm_state + k * kPartial;
              const float wgt = exp2f(sk[0] - M);  // 0 for a half-warp without rows
              L += sk[1] * wgt;
              O += sk[4 + tid] * wgt;
            }
          }
          part[4 + tid] = O;
          if (tid == 0) { part[0] = M; part[1] = L; }
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) {
          const uint32_t prev = atomicAdd(&p.head_done[hq], 1u);
          sm_last = prev + 1u == (uint32_t)nlist;
        }
        __syncthreads();
        if (sm_last) {  // every block of the head has published: merge
          __threadfence();
          if (tid < kDim) {
            float M = -INFINITY;
            for (int k0 = 0; k0 < nlist; k0 += 8) {
              float mv[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                mv[j] = k0 + j < nlist ? __ldcg(p.partial + ((int64_t)(sm_list[k0 + j] + seg.hk) * G + g) * kPartial)
                                       : -INFINITY;
#pragma unroll
              for (int j = 0; j < 8; ++j) M = fmaxf(M, mv[j]);
            }
            float L = 0.0f, O = 0.0f;
            for (int k0 = 0; k0 < nlist; k0 += 8) {
              float mv[8], lv[8], ov[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const bool in = k0 + j < nlist;
                const float* ps = p.partial + (in ? ((int64_t)(sm_list[k0 + j] + seg.hk) * G + g) * kPartial : 0);
                mv[j] = in ? __ldcg(ps) : -INFINITY;
                lv[j] = in ? __ldcg(ps + 1) : 0.0f;
                ov[j] = in ? __ldcg(ps + 4 + tid) : 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                if (mv[j] == -INFINITY) continue;  // a block that kept no token of this head
                const float wgt = exp2f(mv[j] - M);
                L += lv[j] * wgt;
                O += ov[j] * wgt;
              }
            }
            p.out[hq * kDim + tid] = O / L;
          }
          if (tid == 0) p.head_done[hq] = 0u;
        }
        __syncthreads();
      }
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
}

}  // namespace adamas
