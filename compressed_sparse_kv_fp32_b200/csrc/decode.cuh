// One ADAMAS decode step: one thread-block cluster per (sequence, kv head).
//
// Method (ADAMAS long-context sparse attention article, lnwmold.com/news/826806):
// the query is rotated and bucketed like the keys (§2.1, §2.2), every cached
// token is scored by the L1 distance of its 2-bit codes (§2.3), a token budget of
// the best tokens is kept (§5.2) and exact softmax attention runs over their K/V
// rows (the rotation preserves q.k, §2.1, so the exact product uses the original
// vectors).
//
// Work split.  The grid is one cluster of C blocks per (b, kv head); block r of
// the cluster owns the tokens [r*len/C, (r+1)*len/C) of the head.  Nothing is
// exchanged through global memory: the blocks of a head share their histograms
// and partial softmax states through distributed shared memory, so the step has
// no grid-wide wait and no cross-cluster dependency.
//   phase 1  one warp streams the block's packed code rows into a ring of 32 KiB
//            shared-memory stages with bulk asynchronous copies (one full and one
//            empty mbarrier per stage); sixteen warps encode the G query heads of
//            the kv head, then score every row against them (exact L1, two rows
//            per thread per stage), keep the G distances of every token (shared
//            memory, or the workspace when they do not fit) and count them in one
//            385-bin histogram per query head.
//   -- cluster barrier --
//   phase 2  per query head: the C histograms (read from the peers' shared
//            memory) give the threshold T with count(D < T) < k_eff <= count(D <= T)
//            and, for every distance d, the number of tokens of the head with a
//            smaller distance plus the number of tokens with distance d in
//            lower-ranked blocks.  Pass 1: each warp counts, per distance, the
//            tokens of its slice with D <= T.  Pass 2: each warp scans its slice
//            again in index order and puts every candidate straight at its final
//            slot of the (D, index)-ordered output: slot = #smaller D in the head
//            + #equal D in lower blocks + #equal D in lower warps + #equal D in
//            lower lanes (a warp match).  Slots >= k_eff are dropped, which keeps
//            ties at T for the lowest indices.  The kept rows are then gathered
//            straight into registers (each half-warp keeps four K and four V rows
//            in flight) and folded into an online-softmax state per half-warp;
//            the states become one partial (m, l, o) per query head and block.
//   -- cluster barrier --
//   merge    block 0 of the cluster combines the C partial states of each query
//            head (peers' shared memory) into out and pads idx with -1.
//   -- cluster barrier -- (no block leaves while a peer may still read it)
//
// Every mbarrier wait is bounded: after kWaitLimit polls it sets
// ADAMAS_DEVERR_TIMEOUT and goes on, so every thread still reaches every
// cluster barrier.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

namespace cg = cooperative_groups;

constexpr int kWorkers = 512;                         // scoring / select / gather threads
constexpr int kWorkerWarps = kWorkers / 32;
constexpr int kThreads = kWorkers + 32;               // + the warp that issues the bulk copies
constexpr int kStageRows = 1024;                      // code rows per ring stage
constexpr uint32_t kStageBytes = kStageRows * kCodeBytes;  // 32 KiB
constexpr int kRowsPerThread = kStageRows / kWorkers;
constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
constexpr int kMaxCluster = 16;
constexpr int kHistStride = 388;                      // >= kBins, multiple of 4
constexpr int kPartial = 132;                         // m, l, pad, pad, o[128]
constexpr int kScratch = 256;                         // candidate entries per warp per 256-position group
constexpr int kMaxKept = 2048;                        // kept tokens listed per sweep
constexpr int kGatherRows = 4;                        // K/V rows in flight per half-warp
constexpr uint32_t kWaitLimit = 1u << 20;             // mbarrier polls (about a second)

struct DecodeParams {
  const uint16_t* q;
  const uint8_t* codes;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* seq_lens;
  float* out;
  int32_t* idx;
  uint32_t* err;        // device error word
  uint16_t* dglobal;    // [grid][G][dstride] when distances do not fit in shared memory
  int B, Hq, Hkv;
  int64_t Nmax;
  int budget;
  int cluster;          // blocks per (b, kv head)
  int nstages;          // ring stages, kMinStages..kMaxStages
  int dstride;          // distances per query head and block (>= any block's tokens, multiple of 64)
};

// Shared-memory carve-up (bytes), shared with the host.
//   head:    q codes [G][8], q words + masks [G][16], histograms [G][kHistStride],
//            rank bases [G][kHistStride], partial states [G][kPartial]
//   ring:    nstages x 32 KiB; in phase 2 it holds the per-warp counts
//            [kWorkerWarps][kHistStride] (later the half-warp softmax states),
//            the candidate scratch [kWorkerWarps][kScratch] and the kept list
//   dist:    [G][dstride] u16 when kept in shared memory
struct DecodeSmem {
  static __host__ __device__ inline size_t align128(size_t x) { return (x + 127) / 128 * 128; }
  static __host__ __device__ inline size_t qcodes(int G) { return align128((size_t)G * kCodeWords * 4); }
  static __host__ __device__ inline size_t qconst(int G) { return align128((size_t)G * 2 * kCodeWords * 4); }
  static __host__ __device__ inline size_t hist(int G) { return align128((size_t)G * kHistStride * 4); }
  static __host__ __device__ inline size_t partial(int G) { return align128((size_t)G * kPartial * 4); }
  static __host__ __device__ inline size_t head(int G) {
    return qcodes(G) + qconst(G) + 2 * hist(G) + partial(G);
  }
  static __host__ __device__ inline size_t ring(int nstages) { return (size_t)nstages * kStageBytes; }
  static constexpr __host__ __device__ size_t cnt() { return (size_t)kWorkerWarps * kHistStride * 4; }
  static constexpr __host__ __device__ size_t scratch() { return (size_t)kWorkerWarps * kScratch * 4; }
  static constexpr __host__ __device__ size_t state() { return (size_t)2 * kWorkerWarps * kPartial * 4; }
  static __host__ __device__ inline size_t dist(int G, int dstride, bool in_smem) {
    return in_smem ? align128((size_t)G * dstride * 2) : 0;
  }
  static __host__ __device__ inline size_t total(int G, int nstages, int dstride, bool in_smem) {
    return head(G) + ring(nstages) + dist(G, dstride, in_smem);
  }
};
static_assert(DecodeSmem::cnt() >= DecodeSmem::state(), "softmax states overlay the per-warp counts");
static_assert(DecodeSmem::cnt() + DecodeSmem::scratch() + kMaxKept * 4 <= kMinStages * kStageBytes,
              "phase-2 arrays fit in the smallest ring");

// ------------------------------------------------------------------ block helpers
// Barrier of the sixteen worker warps (the copy warp does not take part).
__device__ __forceinline__ void worker_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kWorkers) : "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Exclusive scan of one int64 per worker thread; returns the prefix and writes the
// total to *total.  Uses sm_tmp[kWorkerWarps + 1].
__device__ __forceinline__ int64_t worker_exclusive_scan(int64_t v, int64_t* sm_tmp, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o *= 2) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm_tmp[warp] = x;
  worker_sync();
  if (warp == 0) {
    int64_t w = lane < kWorkerWarps ? sm_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWorkerWarps) sm_tmp[lane] = w;  // inclusive warp totals
    if (lane == kWorkerWarps - 1) sm_tmp[kWorkerWarps] = w;
  }
  worker_sync();
  const int64_t before = warp > 0 ? sm_tmp[warp - 1] : 0;
  const int64_t res = before + x - v;
  *total = sm_tmp[kWorkerWarps];
  worker_sync();
  return res;
}

// Distances of eight consecutive positions 8*grp .. 8*grp+7 (0xFFFF where grp is
// past the warp's slice).
__device__ __forceinline__ void load_dist8(const uint16_t* drow, int grp, bool in, uint32_t (&d)[8]) {
  uint4 v = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
  if (in) v = *reinterpret_cast<const uint4*>(drow + (size_t)grp * 8);
  d[0] = v.x & 0xFFFFu; d[1] = v.x >> 16; d[2] = v.y & 0xFFFFu; d[3] = v.y >> 16;
  d[4] = v.z & 0xFFFFu; d[5] = v.z >> 16; d[6] = v.w & 0xFFFFu; d[7] = v.w >> 16;
}

// One K/V row (16 bytes of each per lane of a half-warp) folded into the
// half-warp's online-softmax state.  Every lane of the warp calls it (the dot
// product is reduced with shuffles inside the half-warp); `valid` is uniform
// within a half-warp.
__device__ __forceinline__ void softmax_fold(const float (&qf)[8], uint4 kr, uint4 vr, bool valid, float& m_run,
                                             float& l_run, float (&o)[8]) {
  float sc = 0.0f;
  if (valid)
    sc = qf[0] * bf16_lo(kr.x) + qf[1] * bf16_hi(kr.x) + qf[2] * bf16_lo(kr.y) + qf[3] * bf16_hi(kr.y) +
         qf[4] * bf16_lo(kr.z) + qf[5] * bf16_hi(kr.z) + qf[6] * bf16_lo(kr.w) + qf[7] * bf16_hi(kr.w);
  sc += __shfl_xor_sync(0xffffffffu, sc, 8);
  sc += __shfl_xor_sync(0xffffffffu, sc, 4);
  sc += __shfl_xor_sync(0xffffffffu, sc, 2);
  sc += __shfl_xor_sync(0xffffffffu, sc, 1);
  if (!valid) return;
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

// ------------------------------------------------------------------ the kernel
// SMEM_D: the block's distances live in shared memory (else in the workspace).
template <int G, bool SMEM_D>
__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t sm_full[kMaxStages];
  __shared__ __align__(8) uint64_t sm_empty[kMaxStages];
  __shared__ int sm_T[kMaxGroup];
  __shared__ int sm_kept_total;
  __shared__ int sm_wlt[kWorkerWarps];    // per warp: candidates with D < T
  __shared__ int sm_weq[kWorkerWarps];    // per warp: candidates with D == T
  __shared__ int sm_wkept[kWorkerWarps];  // per warp: first position of its kept tokens in the list
  __shared__ int64_t sm_scan[kWorkerWarps + 1];

  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.cluster;
  const int rank = (int)cluster.block_rank();
  const int hk = (int)(blockIdx.x / (unsigned)C);  // (b, kv head) of the cluster
  const int b = hk / p.Hkv, kvh = hk - b * p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool worker = warp < kWorkerWarps;
  const uint32_t lt = (1u << lane) - 1u;

  unsigned char* cur = smem;
  uint32_t* sm_q = reinterpret_cast<uint32_t*>(cur);      cur += DecodeSmem::qcodes(G);   // [G][8]
  uint32_t* sm_qc = reinterpret_cast<uint32_t*>(cur);     cur += DecodeSmem::qconst(G);   // [G][q 8 | m 8]
  uint32_t* sm_hist = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::hist(G);     // [G][kHistStride]
  uint32_t* sm_rank = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::hist(G);     // [G][kHistStride]
  float* sm_part = reinterpret_cast<float*>(cur);         cur += DecodeSmem::partial(G);  // [G][kPartial]
  unsigned char* ring = cur;                              cur += DecodeSmem::ring(p.nstages);
  uint16_t* dist;
  if constexpr (SMEM_D) dist = reinterpret_cast<uint16_t*>(cur);
  else dist = p.dglobal + (size_t)blockIdx.x * G * p.dstride;
  // phase-2 arrays over the ring
  uint32_t* sm_cnt = reinterpret_cast<uint32_t*>(ring);                                    // [kWorkerWarps][kHistStride]
  float* sm_state = reinterpret_cast<float*>(ring);                                        // [2*kWorkerWarps][kPartial]
  uint32_t* sm_scratch = reinterpret_cast<uint32_t*>(ring + DecodeSmem::cnt());            // [kWorkerWarps][kScratch]
  int32_t* sm_kept = reinterpret_cast<int32_t*>(ring + DecodeSmem::cnt() + DecodeSmem::scratch());  // [kMaxKept]

  // ---- the head's length and this block's tokens
  int64_t len_b = p.seq_lens[b];
  if (len_b < 0 || len_b > p.Nmax) {
    if (rank == 0 && tid == 0) atomicOr(p.err, kErrSeqLen);
    len_b = len_b < 0 ? 0 : p.Nmax;
  }
  const int keff = (int)min((int64_t)p.budget, len_b);
  const int64_t t0 = (int64_t)rank * len_b / C;
  const int seg_len = (int)((int64_t)(rank + 1) * len_b / C - t0);  // <= dstride (host sizing)
  const int NS = p.nstages;
  const int nst = keff > 0 ? (seg_len + kStageRows - 1) / kStageRows : 0;  // nothing to score without a budget
  const int64_t kv_base = (int64_t)hk * p.Nmax;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm_full[i], 1);
      mbar_init(&sm_empty[i], kWorkerWarps);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < G * kHistStride; i += kThreads) sm_hist[i] = 0u;
  __syncthreads();

  // ================================================================ phase 1
  if (!worker) {
    if (lane == 0) {
      const unsigned char* src = p.codes + (kv_base + t0) * kCodeBytes;
      for (int i = 0; i < nst; ++i) {
        const int buf = i % NS;
        if (i >= NS && !mbar_wait(&sm_empty[buf], (uint32_t)((i / NS) - 1) & 1u, kWaitLimit))
          atomicOr(p.err, kErrTimeout);
        const uint32_t bytes = (uint32_t)min(kStageRows, seg_len - i * kStageRows) * kCodeBytes;
        mbar_arrive_expect_tx(&sm_full[buf], bytes);
        bulk_copy_g2s(ring + (size_t)buf * kStageBytes, src + (size_t)i * kStageBytes, bytes, &sm_full[buf]);
      }
    }
    __syncwarp();
  } else {
    if (warp < G && keff > 0) {
      const uint32_t w = encode128_warp(p.q + ((int64_t)b * p.Hq + kvh * G + warp) * kDim, lane);
      if (lane < kCodeWords) {
        sm_q[warp * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + kCodeWords + lane] = query_mask(w);
      }
    }
    worker_sync();
    constexpr bool kRegQ = G <= 2;  // query words in registers (else read from shared memory per row)
    uint32_t rq[kRegQ ? G : 1][kCodeWords], rm[kRegQ ? G : 1][kCodeWords];
    if constexpr (kRegQ) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int w = 0; w < kCodeWords; ++w) {
          rq[g][w] = sm_qc[g * 2 * kCodeWords + w];
          rm[g][w] = sm_qc[g * 2 * kCodeWords + kCodeWords + w];
        }
    }
    for (int i = 0; i < nst; ++i) {
      const int buf = i % NS;
      if (!mbar_wait(&sm_full[buf], (uint32_t)(i / NS) & 1u, kWaitLimit)) atomicOr(p.err, kErrTimeout);
      const int rows = min(kStageRows, seg_len - i * kStageRows);
      const unsigned char* st = ring + (size_t)buf * kStageBytes;
#pragma unroll
      for (int j = 0; j < kRowsPerThread; ++j) {
        const int r = j * kWorkers + tid;
        if (r < rows) {
          const uint4 x0 = *reinterpret_cast<const uint4*>(st + (size_t)r * kCodeBytes);
          const uint4 x1 = *reinterpret_cast<const uint4*>(st + (size_t)r * kCodeBytes + 16);
          const uint32_t k[kCodeWords] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t k1[kCodeWords];
          key_shift(k, k1);
          const int t = i * kStageRows + r;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            int d;
            if constexpr (kRegQ) {
              d = l1_distance(k, k1, rq[g], rm[g]);
            } else {
              uint32_t qg[kCodeWords], mg[kCodeWords];
              const uint4* s4 = reinterpret_cast<const uint4*>(sm_qc + g * 2 * kCodeWords);
              const uint4 a0 = s4[0], a1 = s4[1], m0 = s4[2], m1 = s4[3];
              qg[0] = a0.x; qg[1] = a0.y; qg[2] = a0.z; qg[3] = a0.w;
              qg[4] = a1.x; qg[5] = a1.y; qg[6] = a1.z; qg[7] = a1.w;
              mg[0] = m0.x; mg[1] = m0.y; mg[2] = m0.z; mg[3] = m0.w;
              mg[4] = m1.x; mg[5] = m1.y; mg[6] = m1.z; mg[7] = m1.w;
              d = l1_distance(k, k1, qg, mg);
            }
            dist[(size_t)g * p.dstride + t] = (uint16_t)d;
            atomicAdd(&sm_hist[g * kHistStride + d], 1u);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm_empty[buf]);
    }
  }
  __syncthreads();
  cluster.sync();  // every block's histograms are complete and visible to the cluster

  // ================================================================ phase 2
  if (worker && keff > 0) {
    // ---- thresholds and rank bases of every query head (histograms of the whole cluster)
    if (tid < G) sm_T[tid] = kBins - 1;  // always overwritten when the histograms are consistent
    worker_sync();
    for (int g = 0; g < G; ++g) {
      const int d = tid;  // bins 0..kBins-1 on the first kBins threads
      int64_t H = 0, P = 0;
      if (d < kBins) {
        uint32_t v[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          v[r] = r < C ? cluster.map_shared_rank(sm_hist, r)[g * kHistStride + d] : 0u;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          H += v[r];
          if (r < rank) P += v[r];
        }
      }
      int64_t tot;
      const int64_t base = worker_exclusive_scan(H, sm_scan, &tot);
      if (d < kBins) {
        if (base < keff && base + H >= keff) sm_T[g] = d;
        sm_rank[g * kHistStride + d] = (uint32_t)(base + P);
      }
    }
    worker_sync();

    const int hw = tid >> 4, hl = tid & 15;  // 32 half-warps
    const float kScoreScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e)/sqrt(128)
    uint32_t* scr = sm_scratch + warp * kScratch;
    // warp slices over 8-position groups of the block's distances
    const int ngrp = (seg_len + 7) >> 3;
    const int gpw = (ngrp + kWorkerWarps - 1) / kWorkerWarps;
    const int wg0 = min(ngrp, warp * gpw), wg1 = min(ngrp, (warp + 1) * gpw);

    for (int g = 0; g < G; ++g) {
      const int64_t hq = (int64_t)b * p.Hq + kvh * G + g;
      int32_t* idx_h = p.idx + hq * p.budget;
      const uint16_t* drow = dist + (size_t)g * p.dstride;
      const uint32_t* rank_g = sm_rank + g * kHistStride;
      const uint32_t T = (uint32_t)sm_T[g];

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

      // sweeps of at most kMaxKept kept tokens (one sweep unless the block keeps more)
      for (int c0 = 0;; c0 += kMaxKept) {
        for (int i = tid; i < kWorkerWarps * kHistStride; i += kWorkers) sm_cnt[i] = 0u;
        worker_sync();
        // ---- pass 1: per-warp counts of the candidates (D <= T) per distance
        int nlt = 0, neq = 0;
        for (int gb = wg0; gb < wg1; gb += 32) {
          const int grp = gb + lane;
          uint32_t dv[8];
          load_dist8(drow, grp, grp < wg1, dv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int pos = grp * 8 + e;
            if (dv[e] <= T && pos < seg_len) {
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
        worker_sync();
        for (int d = tid; d <= (int)T; d += kWorkers) {  // exclusive prefix over the warps, per distance
          uint32_t run = 0;
          for (int w = 0; w < kWorkerWarps; ++w) {
            const uint32_t cw = sm_cnt[w * kHistStride + d];
            sm_cnt[w * kHistStride + d] = run;
            run += cw;
          }
        }
        if (tid == 0) {  // kept tokens per warp: every D < T, and the ties at T within the quota
          const int tie0 = (int)rank_g[T];
          int ties_before = 0, kept_before = 0;
          for (int w = 0; w < kWorkerWarps; ++w) {
            const int ties = min(max(keff - (tie0 + ties_before), 0), sm_weq[w]);
            sm_wkept[w] = kept_before;
            kept_before += sm_wlt[w] + ties;
            ties_before += sm_weq[w];
          }
          sm_kept_total = kept_before;
        }
        worker_sync();
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
            if (dv[e] <= T && pos < seg_len) mask |= 1u << e;
          }
          const int cnum = __popc(mask);
          if (__ballot_sync(0xffffffffu, cnum != 0) == 0u) continue;
          int incl = cnum;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 *= 2) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o2);
            if (lane >= o2) incl += y;
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          int at = incl - cnum;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (mask & (1u << e)) scr[at++] = (uint32_t)(grp * 8 + e) << 9 | dv[e];
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
              const uint32_t slot = rank_g[d] + sm_cnt[warp * kHistStride + d] + __popc(peers & lt);
              if (slot < (uint32_t)keff) {
                kept = true;
                if (c0 == 0) idx_h[slot] = (int32_t)(t0 + (int64_t)(ent >> 9));
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
        worker_sync();
        // ---- gather the listed rows straight into registers; the trip count depends
        // on the warp only, so both half-warps always reach the shuffles together
        const int n_list = max(0, min(kMaxKept, kept_total - c0));
        for (int rb = 2 * warp; rb < n_list; rb += 2 * kWorkerWarps * kGatherRows) {
          uint4 kr[kGatherRows], vr[kGatherRows];
#pragma unroll
          for (int j = 0; j < kGatherRows; ++j) {
            const int row = rb + 2 * kWorkerWarps * j + (hw & 1);
            kr[j] = make_uint4(0u, 0u, 0u, 0u);
            vr[j] = kr[j];
            if (row < n_list) {
              const int64_t t = t0 + sm_kept[row];
              kr[j] = __ldcg(reinterpret_cast<const uint4*>(p.K + (kv_base + t) * kDim) + hl);
              vr[j] = __ldcg(reinterpret_cast<const uint4*>(p.V + (kv_base + t) * kDim) + hl);
            }
          }
#pragma unroll
          for (int j = 0; j < kGatherRows; ++j) {
            const int row = rb + 2 * kWorkerWarps * j + (hw & 1);
            softmax_fold(qf, kr[j], vr[j], row < n_list, m_run, l_run, o);
          }
        }
        worker_sync();
        if (c0 + kMaxKept >= kept_total) break;
      }
      // ---- half-warp states -> this block's partial state for the query head
      {
        float* st = sm_state + hw * kPartial;
        if (hl == 0) { st[0] = m_run; st[1] = l_run; }
#pragma unroll
        for (int e = 0; e < 8; ++e) st[4 + 8 * hl + e] = o[e];
      }
      worker_sync();
      if (tid < kDim) {
        float M = -INFINITY;
        for (int k = 0; k < 2 * kWorkerWarps; ++k) M = fmaxf(M, sm_state[k * kPartial]);
        float L = 0.0f, O = 0.0f;
        if (M != -INFINITY) {
          for (int k = 0; k < 2 * kWorkerWarps; ++k) {
            const float* sk = sm_state + k * kPartial;
            const float wgt = exp2f(sk[0] - M);  // 0 for a half-warp without rows
            L += sk[1] * wgt;
            O += sk[4 + tid] * wgt;
          }
        }
        sm_part[g * kPartial + 4 + tid] = O;
        if (tid == 0) { sm_part[g * kPartial] = M; sm_part[g * kPartial + 1] = L; }
      }
      worker_sync();
    }
  }
  __syncthreads();
  cluster.sync();  // every block's partial states are complete

  // ================================================================ merge (block 0 of the cluster)
  if (rank == 0 && worker) {
    for (int i = tid; i < G * kDim; i += kWorkers) {
      const int g = i / kDim, e = i - g * kDim;
      const int64_t hq = (int64_t)b * p.Hq + kvh * G + g;
      float res = 0.0f;
      if (keff > 0) {
        float mv[kMaxCluster], lv[kMaxCluster], ov[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          mv[r] = -INFINITY; lv[r] = 0.0f; ov[r] = 0.0f;
          if (r < C) {
            const float* pr = cluster.map_shared_rank(sm_part, r) + g * kPartial;
            mv[r] = pr[0]; lv[r] = pr[1]; ov[r] = pr[4 + e];
          }
        }
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) M = fmaxf(M, mv[r]);
        float L = 0.0f, O = 0.0f;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          if (mv[r] == -INFINITY) continue;  // a block that kept no token of this head
          const float wgt = exp2f(mv[r] - M);
          L += lv[r] * wgt;
          O += ov[r] * wgt;
        }
        res = O / L;
      }
      p.out[hq * kDim + e] = res;
    }
    for (int i = tid; i < G * p.budget; i += kWorkers) {
      const int g = i / p.budget, r = i - g * p.budget;
      if (r >= keff) p.idx[((int64_t)b * p.Hq + kvh * G + g) * p.budget + r] = -1;
    }
  }
  __syncthreads();
  cluster.sync();  // peers may still be reading this block's shared memory until here
}

}  // namespace adamas
