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
//   phase 1  per segment: encode the G query heads of the kv head; stream the
//            segment's packed codes through a ring of 32 KiB shared-memory
//            stages filled by bulk asynchronous copies (cp.async.bulk, one
//            mbarrier per stage, all but one stage in flight); each thread scores
//            two code rows per stage (G distances each), keeps the distances in
//            shared memory and adds them to one 385-bin histogram per query
//            head; the histograms are published to the workspace.
//   -- grid-wide wait --
//   phase 2  per segment and query head: sum the head's histograms (one per
//            segment of that head, loaded together) to get the threshold T with
//            count(D < T) < k_eff <= count(D <= T).  Each warp scans its slice of
//            the distances eight at a time and compacts the tokens with D <= T,
//            in index order, into a list; then every listed token goes straight
//            to its final slot of the (D, index)-ordered output:
//            slot = #tokens with smaller D + #tokens with equal D and a lower
//            index (earlier segments from their histograms, earlier warps from
//            per-warp counts, earlier lanes by a warp match).  Slots >= k_eff are
//            dropped, which keeps ties at T for the lowest indices.  The K and V
//            rows of every kept token are prefetched into L2 on the spot.
//   -- grid-wide wait --
//   phase 3  the kept rows of all query heads form a second range, cut evenly
//            over the blocks; each block stages its rows' K and V in shared
//            memory with 16-byte cp.async copies, every half-warp keeps an
//            online-softmax state over its rows, the block publishes one partial
//            state per query head it touched, and the last block to finish a
//            query head (atomic ticket, no waiting) merges the partials into out.
//
// Every wait is bounded: a grid-wide wait gives up after kSpinLimit polls and a
// stage wait after kMbarLimit polls; either sets ADAMAS_DEVERR_TIMEOUT.
#pragma once

#include "common.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kHistStride = 388;                     // >= kBins, multiple of 4
constexpr int kPartial = 132;                        // m, l, pad, pad, o[128]
constexpr int kRowsPerThread = 2;                    // code rows per thread per stage
constexpr int kStageTokens = kThreads * kRowsPerThread;
constexpr uint32_t kStageBytes = kStageTokens * kCodeBytes;  // 32 KiB
constexpr int kStages = 4;                           // most ring stages (fewer when shared memory is short)
constexpr int kMinStages = 2;
constexpr uint32_t kRowBytes = 2 * kDim * 2;         // one K row + one V row (bf16)
constexpr int kMaxRowsStaged = 512;
constexpr int kMaxBlocks = 1024;
constexpr uint32_t kSpinLimit = 1u << 20;            // grid-wide wait polls (about a second)
constexpr uint32_t kMbarLimit = 1u << 20;            // stage wait polls

struct DecodeParams {
  const uint16_t* q;
  const uint8_t* codes;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* seq_lens;
  float* out;
  int32_t* idx;
  uint32_t* ctrl;       // [0..1] grid-wait word (generation << 32 | arrivals), [2] error word
  uint32_t* head_done;  // [B*Hq] tickets of phase 3
  uint32_t* hist;       // [(S + B*Hkv) * G][kHistStride]
  float* partial;       // [(S + B*Hq)][kPartial]
  uint16_t* dglobal;    // [S][G][dstride] when distances do not fit in shared memory
  int B, Hq, Hkv;
  int64_t Nmax;
  int budget;
  int S;
  int64_t range_cap;    // >= units of any block
  int smem_d;           // distances kept in shared memory
  int row_cap;          // K/V rows staged per chunk in phase 3
  int nstages;          // ring stages in phase 1, kMinStages..kStages
};

// Shared-memory carve-up (bytes), shared with the host.
struct DecodeSmem {
  static __host__ __device__ inline size_t align128(size_t x) { return (x + 127) / 128 * 128; }
  static __host__ __device__ inline size_t meta(int B) { return (size_t)(B + 1) * 16 + (size_t)B * 4; }
  static __host__ __device__ inline size_t qwords(int G) { return (size_t)G * kCodeWords * 4; }
  // histograms (phase 1), per-warp counts + rank bases + round totals (phase 2),
  // half-warp softmax states (phase 3)
  static __host__ __device__ inline size_t work(int G) {
    const int rows = G > kWarps + 2 ? G : kWarps + 2;
    return (size_t)rows * kHistStride * 4;
  }
  static __host__ __device__ inline size_t rowidx() { return (size_t)kMaxRowsStaged * 4; }
  static __host__ __device__ inline size_t ring(int nstages) { return (size_t)nstages * kStageBytes; }
  static __host__ __device__ inline int64_t dstride(int64_t range_cap) { return (range_cap + 63) / 64 * 64; }
  static __host__ __device__ inline size_t dist(int G, int64_t range_cap, bool in_smem) {
    return in_smem ? (size_t)G * (size_t)dstride(range_cap) * 2 : 0;
  }
  static __host__ __device__ inline size_t big(int G, int64_t range_cap, bool in_smem, int nstages) {
    return ring(nstages) + dist(G, range_cap, in_smem);
  }
  static __host__ __device__ inline size_t total(int B, int G, int64_t range_cap, bool in_smem, int nstages) {
    return align128(meta(B)) + align128(qwords(G)) + align128(work(G)) + align128(rowidx()) +
           align128(big(G, range_cap, in_smem, nstages));
  }
  static __host__ __device__ inline int row_cap(int G, int64_t range_cap, bool in_smem, int nstages) {
    const size_t rows = big(G, range_cap, in_smem, nstages) / kRowBytes;
    return (int)(rows < (size_t)kMaxRowsStaged ? rows : (size_t)kMaxRowsStaged);
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

// ------------------------------------------------------------------ the kernel
template <int G>
__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t sm_full[kStages];
  __shared__ int sm_flag;
  __shared__ int sm_T;
  __shared__ int sm_last;
  __shared__ int sm_nlist;
  __shared__ int64_t sm_scan[kWarps + 1];
  __shared__ int sm_list[kMaxBlocks];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, S = p.S, B = p.B;
  const uint32_t lt = (1u << lane) - 1u;

  int64_t* sm_uoff = reinterpret_cast<int64_t*>(smem);                  // [B + 1]
  int64_t* sm_roff = sm_uoff + (B + 1);                                 // [B + 1]
  int32_t* sm_len = reinterpret_cast<int32_t*>(sm_roff + (B + 1));      // [B]
  unsigned char* cur = smem + DecodeSmem::align128(DecodeSmem::meta(B));
  uint32_t* sm_q = reinterpret_cast<uint32_t*>(cur);                    // [G][8]
  cur += DecodeSmem::align128(DecodeSmem::qwords(G));
  uint32_t* sm_work = reinterpret_cast<uint32_t*>(cur);                 // [rows][kHistStride]
  cur += DecodeSmem::align128(DecodeSmem::work(G));
  int32_t* sm_rowidx = reinterpret_cast<int32_t*>(cur);                 // [kMaxRowsStaged]
  cur += DecodeSmem::align128(DecodeSmem::rowidx());
  unsigned char* sm_big = cur;  // phase 1: ring | distances; phase 2: candidate lists | distances; phase 3: rows

  const int nstages = p.nstages;
  const int64_t dstride = DecodeSmem::dstride(p.range_cap);
  uint16_t* dbuf = p.smem_d ? reinterpret_cast<uint16_t*>(sm_big + DecodeSmem::ring(nstages))
                            : p.dglobal + (int64_t)s * G * dstride;

  uint32_t gen0 = 0;
  if (tid == 0) {
    for (int k = 0; k < nstages; ++k) mbar_init(&sm_full[k], 1);
    fence_mbar_init();
    gen0 = (uint32_t)(ld_relaxed_gpu64(reinterpret_cast<const unsigned long long*>(p.ctrl)) >> 32);
  }

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
  uint32_t gstage = 0;  // stages consumed so far by this block (same in every thread)
  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    const unsigned char* src = p.codes + ((int64_t)seg.hk * p.Nmax + seg.t0) * kCodeBytes;
    const int64_t nst = (seg.len + kStageTokens - 1) / kStageTokens;
    auto issue = [&](int64_t i) {
      const uint32_t buf = (gstage + (uint32_t)i) % (uint32_t)nstages;
      const int64_t rows = min((int64_t)kStageTokens, seg.len - i * kStageTokens);
      const uint32_t bytes = (uint32_t)rows * kCodeBytes;
      mbar_arrive_expect_tx(&sm_full[buf], bytes);
      bulk_copy_g2s(sm_big + buf * kStageBytes, src + i * kStageBytes, bytes, &sm_full[buf]);
    };
    if (tid == 0) {
      fence_proxy_async_smem();
      for (int64_t i = 0; i < min(nst, (int64_t)nstages - 1); ++i) issue(i);
    }
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

    for (int64_t i = 0; i < nst; ++i) {
      if (tid == 0 && i + nstages - 1 < nst) {
        fence_proxy_async_smem();
        issue(i + nstages - 1);
      }
      const uint32_t gs = gstage + (uint32_t)i;
      const uint32_t buf = gs % (uint32_t)nstages;
      if (!mbar_wait(&sm_full[buf], (gs / (uint32_t)nstages) & 1u, kMbarLimit)) atomicOr(p.ctrl + 2, kErrTimeout);
      const unsigned char* stage = sm_big + buf * kStageBytes;
#pragma unroll
      for (int j = 0; j < kRowsPerThread; ++j) {
        const int r = j * kThreads + tid;
        const int64_t t = i * kStageTokens + r;
        if (t < seg.len) {
          const uint4* row = reinterpret_cast<const uint4*>(stage + r * kCodeBytes);
          const uint4 a = row[0], c = row[1];
          const uint32_t kc[kCodeWords] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
          uint32_t e[kCodeWords];
          key_odd_mask(kc, e);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int d = l1_distance(kc, e, qw[g]);
            dbuf[(int64_t)g * dstride + seg.soff + t] = (uint16_t)d;
            atomicAdd(&sm_work[g * kHistStride + d], 1u);
          }
        }
      }
      __syncthreads();
    }
    gstage += (uint32_t)nst;
    for (int i = tid; i < G * kBins; i += kThreads) {
      const int g = i / kBins, d = i - g * kBins;
      p.hist[((int64_t)(s + seg.hk) * G + g) * kHistStride + d] = sm_work[g * kHistStride + d];
    }
    __syncthreads();
    u += seg.len;
  }

  if (!grid_wait(p.ctrl, S, gen0, &sm_flag)) return;

  // ================================================================ phase 2
  uint32_t* sm_cnt = sm_work;                                // [kWarps][kHistStride]
  uint32_t* sm_rank = sm_work + kWarps * kHistStride;        // [kHistStride]
  uint32_t* sm_round = sm_work + (kWarps + 1) * kHistStride; // [kHistStride]
  uint32_t* cand = reinterpret_cast<uint32_t*>(sm_big);      // per-warp lists over the idle ring
  const int cap_w = (int)(DecodeSmem::ring(nstages) / 4 / kWarps);
  const int64_t round_tokens = (int64_t)kWarps * (cap_w - 32) / 8 * 8;
  uint32_t* my_list = cand + warp * cap_w;
  for (int64_t u = u_lo; u < u_hi;) {
    const Segment seg = segment_at(u, u_lo, u_hi, sm_uoff, sm_len, B, p.Hkv);
    const int64_t len_b = sm_len[seg.b];
    const int keff = (int)min((int64_t)p.budget, len_b);
    if (keff > 0) {
      if (warp == 0) {
        const int n = list_blocks(owner_of(seg.head_u0, U, S), owner_of(seg.head_u0 + len_b - 1, U, S), U, S,
                                  sm_list);
        if (lane == 0) sm_nlist = n;
      }
      __syncthreads();
      const int nlist = sm_nlist;
      const bool first_segment = sm_list[0] == s;
      const int64_t kv_base = (int64_t)seg.hk * p.Nmax;
      for (int g = 0; g < G; ++g) {
        const int64_t hq = (int64_t)seg.b * p.Hq + seg.kvh * G + g;
        int32_t* idx_h = p.idx + hq * p.budget;
        // ---- threshold and rank bases from the head's histograms
        int64_t H = 0, P = 0;
        if (tid < kBins) {
          for (int k0 = 0; k0 < nlist; k0 += 8) {
            uint32_t v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              v[j] = k0 + j < nlist
                         ? __ldcg(&p.hist[((int64_t)(sm_list[k0 + j] + seg.hk) * G + g) * kHistStride + tid])
                         : 0u;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              H += v[j];
              if (k0 + j < nlist && sm_list[k0 + j] < s) P += v[j];
            }
          }
        }
        int64_t tot;
        const int64_t base = block_exclusive_scan(H, sm_scan, &tot);
        if (tid < kBins) {
          if (base < keff && base + H >= keff) sm_T = tid;
          sm_rank[tid] = (uint32_t)(base + P);
        }
        __syncthreads();
        const int T = sm_T;
        const uint16_t* drow = dbuf + (int64_t)g * dstride;
        // ---- rounds over slices of the segment, in index order
        for (int64_t r0 = 0; r0 < seg.len; r0 += round_tokens) {
          const int64_t a0 = seg.soff + r0, a1 = seg.soff + min(seg.len, r0 + round_tokens);
          const int64_t grp0 = a0 >> 3, ngrp = ((a1 + 7) >> 3) - grp0;
          const int64_t gpw = (ngrp + kWarps - 1) / kWarps;
          const int64_t wg0 = grp0 + min(ngrp, (int64_t)warp * gpw), wg1 = grp0 + min(ngrp, (int64_t)(warp + 1) * gpw);
          for (int i = tid; i < kWarps * kHistStride; i += kThreads) sm_cnt[i] = 0u;
          __syncthreads();
          // compaction: tokens with D <= T, in index order, into this warp's list
          int n_w = 0;
          for (int64_t gb = wg0; gb < wg1; gb += 32) {
            const int64_t grp = gb + lane;
            uint4 v = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
            if (grp < wg1) v = *reinterpret_cast<const uint4*>(drow + grp * 8);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            uint32_t mask = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int64_t pos = grp * 8 + e;
              const uint32_t d = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
              if (grp < wg1 && pos >= a0 && pos < a1 && d <= (uint32_t)T) mask |= 1u << e;
            }
            const int c = __popc(mask);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o *= 2) {
              const int y = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += y;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            int at = n_w + incl - c;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (mask & (1u << e)) {
                const uint32_t d = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                my_list[at++] = (uint32_t)(grp * 8 + e - seg.soff) << 9 | d;
              }
            }
            n_w += total;
          }
          // per-warp counts per distance, then exclusive prefix over the warps
          for (int k = lane; k < n_w; k += 32) atomicAdd(&sm_cnt[warp * kHistStride + (my_list[k] & 511u)], 1u);
          __syncthreads();
          if (tid <= T) {
            uint32_t run = 0;
            for (int w = 0; w < kWarps; ++w) {
              const uint32_t c = sm_cnt[w * kHistStride + tid];
              sm_cnt[w * kHistStride + tid] = run;
              run += c;
            }
            sm_round[tid] = run;
          }
          __syncthreads();
          // placement, in index order within the warp's list
          for (int k0 = 0; k0 < n_w; k0 += 32) {
            const int k = k0 + lane;
            const bool valid = k < n_w;
            const uint32_t ent = valid ? my_list[k] : 0u;
            const int d = (int)(ent & 511u);
            const uint32_t m = __ballot_sync(0xffffffffu, valid);
            uint32_t peers = 0;
            if (valid) {
              peers = __match_any_sync(m, d);
              const uint32_t slot = sm_rank[d] + sm_cnt[warp * kHistStride + d] + __popc(peers & lt);
              if (slot < (uint32_t)keff) {
                const int64_t t = seg.t0 + (int64_t)(ent >> 9);
                idx_h[slot] = (int32_t)t;
                const uint16_t* kr = p.K + (kv_base + t) * kDim;
                const uint16_t* vr = p.V + (kv_base + t) * kDim;
                prefetch_l2_keep(kr);
                prefetch_l2_keep(kr + 64);
                prefetch_l2_keep(vr);
                prefetch_l2_keep(vr + 64);
              }
            }
            __syncwarp();
            if (valid && (peers & lt) == 0u) sm_cnt[warp * kHistStride + d] += __popc(peers);
            __syncwarp();
          }
          __syncthreads();
          if (tid <= T) sm_rank[tid] += sm_round[tid];
          __syncthreads();
        }
        if (first_segment)
          for (int r = keff + tid; r < p.budget; r += kThreads) idx_h[r] = -1;
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

  if (!grid_wait(p.ctrl, S, gen0 + 1u, &sm_flag)) return;

  // ================================================================ phase 3
  const int64_t R = roff_total;
  const int64_t r_lo = R > 0 ? range_begin(s, R, S) : 0;
  const int64_t r_hi = R > 0 ? range_begin(s + 1, R, S) : 0;
  float* sm_state = reinterpret_cast<float*>(sm_work);   // [2*kWarps][kPartial]
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
    for (int64_t c0 = 0; c0 < slen; c0 += p.row_cap) {
      const int n = (int)min((int64_t)p.row_cap, slen - c0);
      for (int i = tid; i < n; i += kThreads) {
        int32_t t = __ldcg(idx_h + c0 + i);
        if (t < 0 || t >= len_b) t = -1;  // never read outside the sequence
        sm_rowidx[i] = t;
      }
      __syncthreads();
      // every thread copies 16-byte pieces: 16 pieces of K then 16 of V per row
      for (int c = tid; c < n * 32; c += kThreads) {
        const int row = c >> 5, piece = c & 31;
        const int32_t t = sm_rowidx[row];
        if (t >= 0) {
          const uint16_t* srcp = (piece < 16 ? p.K : p.V) + (kv_base + t) * kDim + (piece & 15) * 8;
          cp_async16(sm_big + (size_t)row * kRowBytes + piece * 16, srcp);
        }
      }
      cp_async_wait_all();
      __syncthreads();
      // The trip count depends on the warp only, so both half-warps always reach
      // the full-warp shuffles below together.
      for (int rb = 2 * warp; rb < n; rb += 2 * kWarps) {
        const int row = rb + (hw & 1);
        const bool valid = row < n && sm_rowidx[row] >= 0;
        float sc = 0.0f;
        uint4 vr = make_uint4(0, 0, 0, 0);
        if (valid) {
          const uint4 kr = *reinterpret_cast<const uint4*>(sm_big + (size_t)row * kRowBytes + 16 * hl);
          vr = *reinterpret_cast<const uint4*>(sm_big + (size_t)row * kRowBytes + kDim * 2 + 16 * hl);
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
    // half-warp states -> block partial
    float* st = sm_state + hw * kPartial;
    if (hl == 0) { st[0] = m_run; st[1] = l_run; }
#pragma unroll
    for (int e = 0; e < 8; ++e) st[4 + 8 * hl + e] = o[e];
    if (warp == 0) {
      const int n = list_blocks(owner_of(head_r0, R, S), owner_of(head_r0 + keff - 1, R, S), R, S, sm_list);
      if (lane == 0) sm_nlist = n;
    }
    __syncthreads();
    const int nlist = sm_nlist;
    float* part = p.partial + (s + hq) * kPartial;
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
    if (tid == 0) {
      const uint32_t prev = atomicAdd(&p.head_done[hq], 1u);
      sm_last = prev + 1u == (uint32_t)nlist;
    }
    __syncthreads();
    if (sm_last) {
      __threadfence();
      if (tid < kDim) {
        float M = -INFINITY;
        for (int k0 = 0; k0 < nlist; k0 += 8) {
          float mv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mv[j] = k0 + j < nlist ? __ldcg(p.partial + (sm_list[k0 + j] + hq) * kPartial) : -INFINITY;
#pragma unroll
          for (int j = 0; j < 8; ++j) M = fmaxf(M, mv[j]);
        }
        float L = 0.0f, O = 0.0f;
        for (int k0 = 0; k0 < nlist; k0 += 8) {
          float mv[8], lv[8], ov[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const bool in = k0 + j < nlist;
            const float* ps = p.partial + (in ? (sm_list[k0 + j] + hq) * kPartial : 0);
            mv[j] = in ? __ldcg(ps) : -INFINITY;
            lv[j] = in ? __ldcg(ps + 1) : 0.0f;
            ov[j] = in ? __ldcg(ps + 4 + tid) : 0.0f;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
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
    r += slen;
  }
}

}  // namespace adamas
