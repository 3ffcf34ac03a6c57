// The plain decode step (contiguous cache, per-head selection, no forced rows, no
// rows written by the launch): the path a decode loop takes by default, kept as its
// own kernel so that none of the options' code reaches it.  The step with options
// is decode_step_ext_kernel (decode_ext.cuh).
#pragma once

#include "decode.cuh"

namespace adamas {

// ------------------------------------------------------------------ the kernel
// SMEM_D: the block's distances live in shared memory (else in the workspace).
template <int G, bool SMEM_D>
__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t sm_full[kMaxStages];
  __shared__ __align__(8) uint64_t sm_empty[kMaxStages];
  __shared__ int sm_T[kMaxGroup];
  __shared__ int sm_wlt[kWorkerWarps];  // per warp: candidates with D < T
  __shared__ int sm_weq[kWorkerWarps];  // per warp: candidates with D == T
  __shared__ int sm_wmax[kWorkerWarps];
  __shared__ uint32_t sm_acode[kCodeWords];  // the appended key's code
  __shared__ long long sm_tmp[kWorkerWarps];

  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.cluster;
  const int rank = (int)cluster.block_rank();
  const int hk = (int)(blockIdx.x / (unsigned)C);  // (b, kv head) of the cluster
  const int b = hk / p.Hkv, kvh = hk - b * p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool worker = warp < kWorkerWarps;
  const uint32_t lt = (1u << lane) - 1u;
  const bool push_hist = DecodeSmem::push_hist(G, C);

  unsigned char* cur = smem;
  uint32_t* sm_q = reinterpret_cast<uint32_t*>(cur);      cur += DecodeSmem::qcodes(G);    // [G][8]
  uint32_t* sm_qc = reinterpret_cast<uint32_t*>(cur);     cur += DecodeSmem::qconst(G);    // [G][q 8 | m 8]
  uint32_t* sm_hist = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::hist(G);      // [G][kHistStride]
  uint32_t* sm_rank = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::hist(G);      // [G][kHistStride]
  uint32_t* sm_lpre = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::hist(G);      // [G][kHistStride]
  uint32_t* sm_htab = reinterpret_cast<uint32_t*>(cur);   cur += DecodeSmem::htab(G, C);   // [C][G][kHistStride]
  float* sm_ptab = reinterpret_cast<float*>(cur);         cur += DecodeSmem::ptab(G, C);   // [owned*C][kPartial]
  unsigned char* ring = cur;                              cur += DecodeSmem::ring(p.nstages);
  uint16_t* dist;
  if constexpr (SMEM_D) {
    dist = reinterpret_cast<uint16_t*>(cur);
    cur += DecodeSmem::dist(G, p.dstride, true);
  } else {
    dist = p.dglobal + (size_t)blockIdx.x * G * p.dstride;
  }
  // phase-2 arrays over the ring
  uint32_t* sm_cnt = reinterpret_cast<uint32_t*>(ring);                          // [kWorkerWarps][kHistStride]
  float* sm_state = reinterpret_cast<float*>(ring);                              // [2*kWorkerWarps][kPartial]
  uint32_t* sm_carry = reinterpret_cast<uint32_t*>(ring + DecodeSmem::cnt());    // [kHistStride]
  int32_t* sm_list = reinterpret_cast<int32_t*>(ring + DecodeSmem::cnt() + DecodeSmem::carry());  // [kListCap]
  int32_t* sm_kept = sm_list + kListCap;                                         // [kKeptCap]

  // The next kernel of the stream may be scheduled at once: it waits here, before
  // its first global read or write, until the kernels before it are done.
  grid_launch_dependents();
  grid_dependency_wait();

  // ---- the head's length and this block's tokens (both loads in flight together)
  const int32_t* ap_src = p.append_pos ? p.append_pos + b : p.seq_lens + b;
  int64_t len_b = p.seq_lens[b];
  const int32_t ap_raw = *ap_src;
  const int64_t ap = p.append_pos ? ap_raw : -1;
  if (len_b < 0 || len_b > p.Nmax) {
    if (rank == 0 && tid == 0) atomicOr(p.err, kErrSeqLen);
    len_b = len_b < 0 ? 0 : p.Nmax;
  }
  const int keff = (int)min((int64_t)p.budget, len_b);
  const int64_t t0 = (int64_t)rank * len_b / C;
  int seg_len = (int)((int64_t)(rank + 1) * len_b / C - t0);  // <= dstride by the host's sizing
  if (seg_len > p.dstride) {  // never with the host's plan; keeps every distance store in bounds
    if (tid == 0) atomicOr(p.err, kErrInternal);
    seg_len = p.dstride;
  }
  const int NS = p.nstages;
  const int nst = keff > 0 ? (seg_len + kStageRows - 1) / kStageRows : 0;  // nothing to score without a budget
  const int64_t kv_base = (int64_t)hk * p.Nmax;
  // appended key of this (b, kv head): encoded by a spare worker warp of the block
  // that owns its position (the last block when it lies past the sequence) while
  // the query is encoded.  The code goes to the cache and to shared memory; the
  // stage copy may carry the cache row's old or new bytes, and the workers score
  // the shared-memory copy in its place.
  int64_t apos = -1;
  int arow = -1;  // its row in this block's segment (-1: not scored here)
  if (ap >= 0 && ap < p.Nmax && ((ap >= t0 && ap < t0 + seg_len) || (rank == C - 1 && ap >= len_b))) {
    apos = ap;
    if (ap >= t0 && ap < t0 + seg_len) arow = (int)(ap - t0);
  }
  const int astage = arow >= 0 ? arow / kStageRows : -1;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm_full[i], 1);
      mbar_init(&sm_empty[i], kWorkerWarps);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < G * kHistStride; i += kThreads) sm_hist[i] = 0u;
  if (tid < kMaxGroup) sm_T[tid] = kBins - 1;  // always overwritten when the histograms are consistent

  __syncthreads();
  // Every block of the cluster has started (and may be written to through
  // distributed shared memory) once every thread has arrived here; each thread
  // waits on it before its first such access.
  cluster_arrive();

  // ================================================================ phase 1
  if (!worker) {
    const unsigned char* src = p.codes + (kv_base + t0) * kCodeBytes;
    auto issue = [&](int i) {
      const int buf = i % NS;
      if (i >= NS && !mbar_wait(&sm_empty[buf], (uint32_t)((i / NS) - 1) & 1u, kWaitLimit))
        atomicOr(p.err, kErrTimeout);
      const uint32_t bytes = (uint32_t)min(kStageRows, seg_len - i * kStageRows) * kCodeBytes;
      mbar_arrive_expect_tx(&sm_full[buf], bytes);
      bulk_copy_g2s(ring + (size_t)buf * kStageBytes, src + (size_t)i * kStageBytes, bytes, &sm_full[buf]);
    };
    if (lane == 0)
      for (int i = 0; i < nst; ++i) issue(i);
    __syncwarp();
    cluster_wait();
  } else {
    if (warp < G && keff > 0) {
      const uint32_t w = encode128_warp(p.q + ((int64_t)b * p.Hq + kvh * G + warp) * kDim, lane);
      if (lane < kCodeWords) {
        sm_q[warp * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + kCodeWords + lane] = query_mask(w);
      }
    }
    if (warp == kWorkerWarps - 1 && apos >= 0) {  // the same encoder as adamas_encode_keys
      const uint32_t w = encode128_warp(p.K + (kv_base + apos) * kDim, lane);
      if (lane < kCodeWords) {
        sm_acode[lane] = w;
        reinterpret_cast<uint32_t*>(p.codes_w + (kv_base + apos) * kCodeBytes)[lane] = w;
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
      uint4 kx[kRowsPerThread][2];
#pragma unroll
      for (int j = 0; j < kRowsPerThread; ++j) {
        const int r = j * kWorkers + tid;
        kx[j][0] = make_uint4(0u, 0u, 0u, 0u);
        kx[j][1] = kx[j][0];
        if (r < rows) {
          const uint32_t ra = smem_addr(st + (size_t)r * kCodeBytes);
          kx[j][0] = lds128(ra);
          kx[j][1] = lds128(ra + 16);
        }
      }
      if (i == astage) {  // the appended row: its fresh code
#pragma unroll
        for (int j = 0; j < kRowsPerThread; ++j)
          if (i * kStageRows + j * kWorkers + tid == arow) {
            kx[j][0] = make_uint4(sm_acode[0], sm_acode[1], sm_acode[2], sm_acode[3]);
            kx[j][1] = make_uint4(sm_acode[4], sm_acode[5], sm_acode[6], sm_acode[7]);
          }
      }
#pragma unroll
      for (int j = 0; j < kRowsPerThread; ++j) {
        const int r = j * kWorkers + tid;
        const int t = i * kStageRows + r;
        if (r < rows) {
          const uint4 x0 = kx[j][0], x1 = kx[j][1];
          const uint32_t k[kCodeWords] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t k1[kCodeWords];
          key_shift(k, k1);
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
            if constexpr (SMEM_D) sts16(smem_addr(dist + (size_t)g * p.dstride + t), (uint16_t)d);
            else dist[(size_t)g * p.dstride + t] = (uint16_t)d;
            atomicAdd(&sm_hist[g * kHistStride + d], 1u);
          }
        }
      }
      // Every lane has used its rows: only now does the stage go back to the copy warp
      // (one arrive per warp after __syncwarp does not order other lanes' loads that
      // are still in flight against the refill).
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm_empty[buf]);
    }

    cluster_wait();
    if (push_hist && keff > 0) {  // own histograms into every block's table (row `rank`)
      worker_sync();
      for (int r = 0; r < C; ++r) {
        uint32_t* tab = cluster.map_shared_rank(sm_htab, r) + (size_t)rank * G * kHistStride;
        for (int i = tid; i < G * kHistStride; i += kWorkers) tab[i] = sm_hist[i];
      }
    }
  }
  __syncthreads();
  cluster.sync();  // every block's histograms are complete and visible to the cluster

  // ================================================================ phase 2
  if (worker && keff > 0) {
    // ---- the tail of the last 8-position group of every distance row reads as "far"
    if (tid < G)
      for (int pos = seg_len; pos < ((seg_len + 7) & ~7); ++pos) {
        if constexpr (SMEM_D) sts16(smem_addr(dist + (size_t)tid * p.dstride + pos), 0xFFFFu);
        else dist[(size_t)tid * p.dstride + pos] = 0xFFFFu;
      }
    // ---- thresholds, rank bases and own prefixes of every query head
    for (int g = 0; g < G; ++g) {
      const int d = tid;  // bins 0..kBins-1 on the first kBins threads
      long long H = 0, P = 0, own = 0;
      if (d < kBins) {
        uint32_t v[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          v[r] = 0u;
          if (r < C)
            v[r] = push_hist ? sm_htab[((size_t)r * G + g) * kHistStride + d]
                             : cluster.map_shared_rank(sm_hist, r)[g * kHistStride + d];
        }
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          H += v[r];
          if (r < rank) P += v[r];
        }
        own = sm_hist[g * kHistStride + d];
      }
      // both prefixes in one scan: totals of the head in the high word, own counts in the low one
      const long long pre = worker_exclusive_scan(H << 32 | own, sm_tmp);
      const int base = (int)(pre >> 32);
      if (d < kBins) {
        if (base < keff && base + H >= keff) sm_T[g] = d;
        sm_rank[g * kHistStride + d] = (uint32_t)(base + P);
        sm_lpre[g * kHistStride + d] = (uint32_t)(pre & 0xFFFFFFFFll);
      }
    }
    worker_sync();

    const int hw = tid >> 4, hl = tid & 15;  // two half-warps per worker warp
    const float kScoreScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e)/sqrt(128)
    // warp slices over 8-position groups of the block's distances (full scans)
    const int ngrp = (seg_len + 7) >> 3;
    const int gpw = (ngrp + kWorkerWarps - 1) / kWorkerWarps;
    const int wg0 = min(ngrp, warp * gpw), wg1 = min(ngrp, (warp + 1) * gpw);

    for (int g = 0; g < G; ++g) {
      const int64_t hq = (int64_t)b * p.Hq + kvh * G + g;
      int32_t* idx_h = p.idx + hq * p.budget;
      const uint16_t* drow = dist + (size_t)g * p.dstride;
      const uint32_t* rank_g = sm_rank + g * kHistStride;
      const uint32_t* lpre_g = sm_lpre + g * kHistStride;
      const uint32_t* hist_g = sm_hist + g * kHistStride;
      const uint32_t T = (uint32_t)sm_T[g];
      const int tie_base = (int)rank_g[T];              // output slot of this block's first tie
      const int tie_quota = max(0, keff - tie_base);    // ties this block keeps (its first ones)
      const int n_lt = (int)lpre_g[T];                  // tokens of the block with D < T
      const int n_eq = (int)hist_g[T];                  // ties of the block
      const int n_kept = n_lt + min(tie_quota, n_eq);   // kept tokens, in slot order at [0, n_kept)
      const uint4 qraw = *reinterpret_cast<const uint4*>(p.q + hq * kDim + 8 * hl);

      // The compact path: every token with D <= T (typically a few hundred) is listed
      // in index order, then ranked among the listed tokens of its distance; else the
      // two scans.
      bool compact = n_lt + n_eq <= kListCap && n_kept <= kKeptCap;

      float qf[8];
      float m_run = -INFINITY, l_run = 0.0f, o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = 0.0f;

      // gather of the kept tokens [0, n) of one window into the softmax state
      auto gather = [&](int n, bool prefetch) {
        for (int i = tid; prefetch && i < 4 * n; i += kWorkers) {  // every kept row on its way into L2
          const int64_t t = kv_base + t0 + (int64_t)lds32(smem_addr(sm_kept + (i >> 2)));
          prefetch_l2((i & 2 ? p.V : p.K) + t * kDim + (i & 1) * 64);
        }
        for (int rb = 2 * warp; rb < n; rb += kGatherBatch) {
          uint4 kr[kGatherRows], vr[kGatherRows];
          gather_issue_plain(sm_kept, rb, n, hw, hl, p.K, p.V, kv_base + t0, kr, vr);
          gather_fold(rb, n, hw, qf, kr, vr, m_run, l_run, o);
        }
      };

      if (compact) {
        // ---- list: rounds over consecutive spans of at most kWorkers * 8 groups of 8
        // positions; in a round each thread takes a run of at most eight groups (lanes
        // start at different points of the eight so that a warp's loads spread over the
        // banks) and marks D <= T, and after one block scan of the counts writes its
        // tokens -- (D << 23 | offset) -- from its offset on, so the list is in index
        // order.
        const uint32_t t1x2 = (T + 1) | (T + 1) << 16;
        const int rot = lane & 7;
        for (int i = tid; i < kWorkerWarps * kHistStride; i += kWorkers) sm_cnt[i] = 0u;
        for (int i = tid; i < kHistStride; i += kWorkers) sm_carry[i] = 0u;
        int listed = 0;  // tokens listed by earlier rounds
        for (int r0 = 0; r0 < ngrp; r0 += kWorkers * 8) {
          const int span = min(kWorkers * 8, ngrp - r0);
          const int cnt = (span + kWorkers - 1) / kWorkers;
          const int g0 = r0 + tid * cnt;
          unsigned long long cm = 0ull;  // bit 8j + e: position (g0 + j) * 8 + e
#pragma unroll
          for (int h = 0; h < 8; h += 2) {
            uint4 v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int j = (h + u + rot) & 7, grp = g0 + j;
              v[u] = (j < cnt && grp < r0 + span) ? load_dist8<SMEM_D>(drow, grp)
                                                  : make_uint4(~0u, ~0u, ~0u, ~0u);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) cm |= (unsigned long long)le_bits(v[u], t1x2) << (8 * ((h + u + rot) & 7));
          }
          const int mine = __popcll((long long)cm);
          const uint32_t before = worker_exclusive_scan32((uint32_t)mine, reinterpret_cast<uint32_t*>(sm_tmp));
          if (tid == kWorkers - 1) sm_wmax[0] = (int)before + mine;
          int at = listed + (int)before;
          for (; cm != 0ull; cm &= cm - 1ull, ++at) {
            const int bit = __ffsll((long long)cm) - 1;
            const uint32_t pos = (uint32_t)((g0 + (bit >> 3)) * 8 + (bit & 7));
            const uint32_t dd = load_dist1<SMEM_D>(drow, (int)pos);
            if (at < kListCap) sm_list[at] = (int32_t)(dd << 23 | pos);
          }
          worker_sync();  // the round's total is visible
          listed += sm_wmax[0];
          worker_sync();  // every thread has read it before the next round overwrites it
        }
        if (listed != n_lt + n_eq) {  // never with consistent histograms
          if (tid == 0) atomicOr(p.err, kErrInternal);
          listed = min(listed, kListCap);
        }
        // ---- slots: a token's rank among the block's tokens of its distance is the
        // number of listed tokens of that distance before it (the list is in index
        // order): per round of kWorkers entries, a warp match gives the rank inside the
        // warp, per-warp counts give the warps before, carried counts the rounds before
        for (int r0 = 0; r0 < listed; r0 += kWorkers) {
          const int i = r0 + tid;
          const bool valid = i < listed;
          const uint32_t ent = valid ? lds32(smem_addr(sm_list + i)) : 0u;
          const uint32_t d = ent >> 23, tpos = ent & kPosMask;
          const uint32_t vm = __ballot_sync(0xffffffffu, valid);
          uint32_t peers = 0u;
          if (valid) {
            peers = __match_any_sync(vm, d);
            if ((peers & lt) == 0u) sm_cnt[warp * kHistStride + d] = (uint32_t)__popc(peers);
          }
          worker_sync();
          if (valid) {
            const uint32_t ca = smem_addr(sm_cnt + d);
            uint32_t before = lds32(smem_addr(sm_carry + d)) + (uint32_t)__popc(peers & lt);
#pragma unroll
            for (int w = 0; w < kWorkerWarps - 1; ++w)
              if (w < warp) before += lds32(ca + w * kHistStride * 4);
            const uint32_t slot = rank_g[d] + before;
            const uint32_t kp = lpre_g[d] + before;
            if (slot < (uint32_t)keff && kp < (uint32_t)n_kept) {
              idx_h[slot] = (int32_t)(t0 + tpos);
              sm_kept[kp] = (int32_t)tpos;
            }
          }
          if (r0 + kWorkers < listed) {  // counts carried to the next round
            worker_sync();
            for (int dd = tid; dd < kBins; dd += kWorkers) {
              uint32_t c = 0u;
              for (int w = 0; w < kWorkerWarps; ++w) {
                c += sm_cnt[w * kHistStride + dd];
                sm_cnt[w * kHistStride + dd] = 0u;
              }
              sm_carry[dd] += c;
            }
          }
          worker_sync();
        }
        qf[0] = bf16_lo(qraw.x) * kScoreScale; qf[1] = bf16_hi(qraw.x) * kScoreScale;
        qf[2] = bf16_lo(qraw.y) * kScoreScale; qf[3] = bf16_hi(qraw.y) * kScoreScale;
        qf[4] = bf16_lo(qraw.z) * kScoreScale; qf[5] = bf16_hi(qraw.z) * kScoreScale;
        qf[6] = bf16_lo(qraw.w) * kScoreScale; qf[7] = bf16_hi(qraw.w) * kScoreScale;
        gather(n_kept, false);
        worker_sync();
      }
      if (!compact) {
        // ---- count pass: candidates per warp
        const uint32_t tx2 = T | T << 16, t1x2 = (T + 1) | (T + 1) << 16;
        int c_lt = 0, c_eq = 0;
        for (int gb0 = wg0; gb0 < wg1; gb0 += 32 * kScanBatch) {
          uint4 v[kScanBatch];
#pragma unroll
          for (int it = 0; it < kScanBatch; ++it) {
            const int grp = gb0 + 32 * it + lane;
            v[it] = grp < wg1 ? load_dist8<SMEM_D>(drow, grp) : make_uint4(~0u, ~0u, ~0u, ~0u);
          }
#pragma unroll
          for (int it = 0; it < kScanBatch; ++it)
            if (any_le(v[it], t1x2)) {
              uint32_t mlt, meq;
              cand_bits(v[it], tx2, t1x2, mlt, meq);
              c_lt += __popc(mlt);
              c_eq += __popc(meq);
            }
        }
        c_lt = __reduce_add_sync(0xffffffffu, c_lt);
        c_eq = __reduce_add_sync(0xffffffffu, c_eq);
        if (lane == 0) {
          sm_wlt[warp] = c_lt;
          sm_weq[warp] = c_eq;
        }
        worker_sync();
        int lt_base = 0, eq_base = 0;
#pragma unroll
        for (int w = 0; w < kWorkerWarps; ++w) {
          lt_base += w < warp ? sm_wlt[w] : 0;
          eq_base += w < warp ? sm_weq[w] : 0;
        }
        qf[0] = bf16_lo(qraw.x) * kScoreScale; qf[1] = bf16_hi(qraw.x) * kScoreScale;
        qf[2] = bf16_lo(qraw.y) * kScoreScale; qf[3] = bf16_hi(qraw.y) * kScoreScale;
        qf[4] = bf16_lo(qraw.z) * kScoreScale; qf[5] = bf16_hi(qraw.z) * kScoreScale;
        qf[6] = bf16_lo(qraw.w) * kScoreScale; qf[7] = bf16_hi(qraw.w) * kScoreScale;

        // windows of kKeptCap kept positions; per window, rounds of kListCap D < T tokens
        for (int c0 = 0; c0 < n_kept; c0 += kKeptCap) {
          const int n_win = min(kKeptCap, n_kept - c0);
          for (int r0 = 0; r0 == 0 || r0 < n_lt; r0 += kListCap) {
            const int n_round = max(0, min(kListCap, n_lt - r0));
            // ---- emit pass: the round's D < T tokens to the list; ties (first round) to their slots
            int lt_run = lt_base, eq_run = eq_base;
            for (int gb0 = wg0; gb0 < wg1; gb0 += 32 * kScanBatch) {
              uint4 v[kScanBatch];
#pragma unroll
              for (int it = 0; it < kScanBatch; ++it) {
                const int grp = gb0 + 32 * it + lane;
                v[it] = grp < wg1 ? load_dist8<SMEM_D>(drow, grp) : make_uint4(~0u, ~0u, ~0u, ~0u);
              }
              uint32_t mlt[kScanBatch], meq[kScanBatch];
              int incl[kScanBatch];
              bool mine = false;
#pragma unroll
              for (int it = 0; it < kScanBatch; ++it) {
                mlt[it] = 0u;
                meq[it] = 0u;
                if (any_le(v[it], t1x2)) cand_bits(v[it], tx2, t1x2, mlt[it], meq[it]);
                incl[it] = __popc(mlt[it]) | __popc(meq[it]) << 16;
                mine |= incl[it] != 0;
              }
              if (__ballot_sync(0xffffffffu, mine) == 0u) continue;
              int own[kScanBatch];
#pragma unroll
              for (int it = 0; it < kScanBatch; ++it) own[it] = incl[it];
#pragma unroll
              for (int off = 1; off < 32; off *= 2)
#pragma unroll
                for (int it = 0; it < kScanBatch; ++it) {
                  const int y = __shfl_up_sync(0xffffffffu, incl[it], off);
                  if (lane >= off) incl[it] += y;
                }
#pragma unroll
              for (int it = 0; it < kScanBatch; ++it) {
                const int tot = __shfl_sync(0xffffffffu, incl[it], 31);
                if (own[it] != 0) {
                  const int grp = gb0 + 32 * it + lane;
                  int at_lt = lt_run + ((incl[it] - own[it]) & 0xFFFF);
                  int at_eq = eq_run + ((incl[it] - own[it]) >> 16);
                  const uint32_t w[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const uint32_t pos = (uint32_t)(grp * 8 + e);
                    const uint32_t dval = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                    if (mlt[it] & (1u << e)) {
                      const int k = at_lt++ - r0;
                      if (k >= 0 && k < n_round) sm_list[k] = (int32_t)(dval << 23 | pos);
                    }
                    if (r0 == 0 && (meq[it] & (1u << e))) {
                      const int tie = at_eq++;
                      if (tie < tie_quota) {
                        if (c0 == 0) idx_h[tie_base + tie] = (int32_t)(t0 + pos);
                        const int kp = n_lt + tie - c0;
                        if (kp >= 0 && kp < n_win) sm_kept[kp] = (int32_t)pos;
                      }
                    }
                  }
                }
                lt_run += tot & 0xFFFF;
                eq_run += tot >> 16;
              }
            }
            worker_sync();
            // ---- slots of the round's D < T tokens: rank among equal distances by index
            if (r0 == 0)
              for (int i = tid; i < kHistStride; i += kWorkers) sm_carry[i] = 0u;
            for (int i = tid; i < kWorkerWarps * kHistStride; i += kWorkers) sm_cnt[i] = 0u;
            worker_sync();
            for (int q0 = 0; q0 < n_round; q0 += kWorkers) {
              const int i = q0 + tid;
              const bool valid = i < n_round;
              const uint32_t ent = valid ? lds32(smem_addr(sm_list + i)) : 0u;
              const uint32_t d = ent >> 23;
              const uint32_t m = __ballot_sync(0xffffffffu, valid);
              uint32_t peers = 0u;
              if (valid) {
                peers = __match_any_sync(m, d);
                if ((peers & lt) == 0u) sm_cnt[warp * kHistStride + d] = (uint32_t)__popc(peers);
              }
              worker_sync();
              if (valid) {
                const uint32_t ca = smem_addr(sm_cnt + d);
                uint32_t before = lds32(smem_addr(sm_carry + d));
#pragma unroll
                for (int w = 0; w < kWorkerWarps - 1; ++w)
                  if (w < warp) before += lds32(ca + w * kHistStride * 4);
                before += (uint32_t)__popc(peers & lt);  // rank of the token among the block's equal distances
                const uint32_t tpos = ent & kPosMask;
                if (c0 == 0 && rank_g[d] + before < (uint32_t)keff) idx_h[rank_g[d] + before] = (int32_t)(t0 + tpos);
                const int kp = (int)(lpre_g[d] + before) - c0;
                if (kp >= 0 && kp < n_win) sm_kept[kp] = (int32_t)tpos;
              }
              worker_sync();
              for (int dd = tid; dd < kBins; dd += kWorkers) {  // counts carried to later entries
                uint32_t s = 0u;
                for (int w = 0; w < kWorkerWarps; ++w) {
                  s += sm_cnt[w * kHistStride + dd];
                  sm_cnt[w * kHistStride + dd] = 0u;
                }
                sm_carry[dd] += s;
              }
              worker_sync();
            }
          }
          gather(n_win, true);
          worker_sync();
        }
      }
      // ---- half-warp states -> this block's partial state -> the head's owner
      {
        // the two half-warps of a warp hold the same slice of dimensions: merge them
        // with shuffles first, then one state per warp goes through shared memory
        const float m_o = __shfl_xor_sync(0xffffffffu, m_run, 16);
        const float l_o = __shfl_xor_sync(0xffffffffu, l_run, 16);
        const float m_new = fmaxf(m_run, m_o);
        const float a = m_run == -INFINITY ? 0.0f : exp2f(m_run - m_new);  // 0 for a half-warp without rows
        const float a_o = m_o == -INFINITY ? 0.0f : exp2f(m_o - m_new);
        float* st = sm_state + warp * kPartial;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float oo = __shfl_xor_sync(0xffffffffu, o[e], 16);
          if (hw % 2 == 0) st[4 + 8 * hl + e] = o[e] * a + oo * a_o;
        }
        if (lane == 0) {
          st[0] = m_new;
          st[1] = l_run * a + l_o * a_o;
        }
      }
      worker_sync();
      if (tid < kDim) {
        float M = -INFINITY;
        for (int k = 0; k < kWorkerWarps; ++k) M = fmaxf(M, sm_state[k * kPartial]);
        float L = 0.0f, O = 0.0f;
        if (M != -INFINITY) {
          for (int k = 0; k < kWorkerWarps; ++k) {
            const float* sk = sm_state + k * kPartial;
            const float wgt = exp2f(sk[0] - M);  // 0 for a half-warp without rows
            L += sk[1] * wgt;
            O += sk[4 + tid] * wgt;
          }
        }
        float* dst = cluster.map_shared_rank(sm_ptab, g % C) + ((size_t)(g / C) * C + rank) * kPartial;
        dst[4 + tid] = O;
        if (tid == 0) { dst[0] = M; dst[1] = L; }
      }
      worker_sync();
    }
  }
  __syncthreads();
  cluster.sync();  // every partial state is in its owner's table

  // ================================================================ merge of the owned query heads
  if (worker) {
    for (int g = rank; g < G; g += C) {
      const int64_t hq = (int64_t)b * p.Hq + kvh * G + g;
      for (int e = tid; e < kDim; e += kWorkers) {
        float res = 0.0f;
        if (keff > 0) {
          const float* tab = sm_ptab + (size_t)(g / C) * C * kPartial;
          float M = -INFINITY;
          for (int r = 0; r < C; ++r) M = fmaxf(M, tab[r * kPartial]);
          float L = 0.0f, O = 0.0f;
          for (int r = 0; r < C; ++r) {
            const float mr = tab[r * kPartial];
            if (mr == -INFINITY) continue;  // a block that kept no token of this head
            const float wgt = exp2f(mr - M);
            L += tab[r * kPartial + 1] * wgt;
            O += tab[r * kPartial + 4 + e] * wgt;
          }
          res = O / L;
        }
        p.out[hq * kDim + e] = res;
      }
    }
    if (rank == 0)
      for (int i = tid; i < G * p.budget; i += kWorkers) {
        const int g = i / p.budget, r = i - g * p.budget;
        if (r >= keff) p.idx[((int64_t)b * p.Hq + kvh * G + g) * p.budget + r] = -1;
      }
  }
}

}  // namespace adamas
