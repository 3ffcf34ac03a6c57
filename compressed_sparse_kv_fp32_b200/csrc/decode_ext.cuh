// The decode step with its options: a paged cache read through a block table,
// forced rows (attention sinks and the recent window), the appended K/V rows
// written by the launch, and group-shared selection for grouped query heads.
// Same structure as the plain step (decode_plain.cuh); see decode.cuh for the
// layout of the work.
#pragma once

#include "decode.cuh"

namespace adamas {

// Kernel modes: the plain step has its own kernel (decode_plain.cuh); this one is
// the general per-head step and the group-shared step, which read the options
// (paged cache, forced rows, rows written by the launch) at run time, and the two
// halves of the sequence-sharded step.
constexpr int kModePlain = 0;
constexpr int kModeGeneral = 1;
constexpr int kModeShared = 2;
// Sequence-sharded step: each GPU holds one contiguous slice of every sequence.
//   kModeShardScore   phase 1 only: the slice's distances go to the workspace, each
//                     block's histograms to the workspace and their sum over the
//                     slice to the exchange buffer.
//   kModeShardAttend  phase 2 and the merge, with the threshold and rank bases taken
//                     from every slice's histograms (the exchange buffers of all
//                     GPUs, gathered in slice order); the output is this slice's
//                     softmax state, and idx holds the global indices of the
//                     slice's kept tokens.
// The histogram exchange makes the selection exactly the one of the whole
// sequence: the slices play the part the blocks of a cluster play inside a GPU.
// With vslices = S > 1 the same two launches split every (b, kv head) of one GPU's
// cache into S slices, one cluster each (more clusters for few long heads): the
// score launch writes slice s's histograms at [s][B][Hq], which is then already
// the gathered buffer of the attend launch, token indices are the cache's own, and
// the attend launch writes slice s's state at [s][B][Hq].
constexpr int kModeShardScore = 3;
constexpr int kModeShardAttend = 4;

// SMEM_D: the block's distances live in shared memory (else in the workspace).
// MODE kModeShared: group-shared selection -- the distances of the G query heads are
// summed per token and one budget of tokens is kept for the kv head, which every
// query head of the group attends over (else each query head selects its own).
template <int G, bool SMEM_D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) decode_step_ext_kernel(const DecodeParams p) {
  constexpr bool SHARED = MODE == kModeShared;
  constexpr bool GENERAL = MODE != kModePlain;
  constexpr bool SCORE_ONLY = MODE == kModeShardScore;
  constexpr bool ATTEND_ONLY = MODE == kModeShardAttend;
  static_assert(!(SCORE_ONLY || ATTEND_ONLY) || !SMEM_D, "the sharded step keeps its distances in the workspace");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t sm_full[kMaxStages];
  __shared__ __align__(8) uint64_t sm_empty[kMaxStages];
  __shared__ int sm_T[kMaxGroup];
  __shared__ int sm_wlt[kWorkerWarps];  // per warp: candidates with D < T
  __shared__ int sm_weq[kWorkerWarps];  // per warp: candidates with D == T
  __shared__ int sm_wmax[kWorkerWarps];
  __shared__ uint32_t sm_acode[kCodeWords];  // the appended key's code
  __shared__ long long sm_tmp[kWorkerWarps];
  __shared__ int sm_round[2];       // totals of one round of the ordered pass
  __shared__ unsigned long long sm_len[2];  // sharded step: tokens of the sequence before this slice, in all

  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.cluster;
  const int rank = (int)cluster.block_rank();
  const int clus = (int)(blockIdx.x / (unsigned)C);  // the cluster
  // slices of one (b, kv head) in this launch (the sharded modes on one GPU)
  const int VS = (SCORE_ONLY || ATTEND_ONLY) && p.vslices > 1 ? p.vslices : 1;
  const int hk = clus / VS, vs = clus - hk * VS;  // (b, kv head) of the cluster, its slice
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
  // k_eff of the sequence (of the whole sequence in the sharded step: set below)
  int keff = (int)min((int64_t)p.budget, len_b);
  const bool forced = GENERAL && (p.n_sink > 0 || p.n_recent > 0);
  // distance bins: [0, 384] per query head, [0, 384 G] summed over a group; one more
  // when forced rows take bin 0
  const int nbins = (SHARED ? 3 * kDim * G + 1 : kBins) + (forced ? 1 : 0);
  // the cluster's tokens [sb0, sb0 + sl) (the whole sequence unless sliced), the block's share of them
  const int64_t sb0 = (int64_t)vs * len_b / VS, sl = (int64_t)(vs + 1) * len_b / VS - sb0;
  const int64_t t0 = sb0 + (int64_t)rank * sl / C;
  int seg_len = (int)(sb0 + (int64_t)(rank + 1) * sl / C - t0);  // <= dstride by the host's sizing
  if (seg_len > p.dstride) {  // never with the host's plan; keeps every distance store in bounds
    if (tid == 0) atomicOr(p.err, kErrInternal);
    seg_len = p.dstride;
  }
  const int NS = p.nstages;
  // nothing to score without a budget; the attend half of the sharded step scores nothing
  const int nst = !ATTEND_ONLY && keff > 0 ? (seg_len + kStageRows - 1) / kStageRows : 0;
  const int64_t kv_base = (int64_t)hk * p.Nmax;
  // appended key of this (b, kv head): encoded by a spare worker warp of the block
  // that owns its position (the last block when it lies past the sequence) while
  // the query is encoded.  The code goes to the cache and to shared memory; the
  // stage copy may carry the cache row's old or new bytes, and the workers score
  // the shared-memory copy in its place.
  int64_t apos = -1;
  int arow = -1;  // its row in this block's segment (-1: not scored here)
  if (ap >= 0 && ap < p.Nmax &&
      ((ap >= t0 && ap < t0 + seg_len) || (rank == C - 1 && vs == VS - 1 && ap >= len_b))) {
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
  if (tid < 2) sm_round[tid] = 0;  // a block without tokens runs no round of the ordered pass
  if (tid < 2) sm_len[tid] = 0ull;

  __syncthreads();
  // Sharded step: the sequence's length and this slice's first index are the
  // histogram totals (every scored token is counted once per query head) of all
  // slices and of the slices before this one.
  int64_t ofs = 0;
  const int srank = VS > 1 ? vs : p.shard_rank, sworld = VS > 1 ? VS : p.shard_world;
  if constexpr (ATTEND_ONLY) {
    const uint32_t* h0 = p.hist_all + ((int64_t)b * p.Hq + (int64_t)kvh * G) * kHistStride;
    const int64_t rs = (int64_t)p.B * p.Hq * kHistStride;
    unsigned long long before = 0ull, total = 0ull;
    for (int i = tid; i < sworld * kBins; i += kThreads) {
      const int r = i / kBins, d = i - r * kBins;
      const uint32_t v = h0[r * rs + d];
      total += v;
      if (r < srank) before += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    if (lane == 0) {
      atomicAdd(&sm_len[0], before);
      atomicAdd(&sm_len[1], total);
    }
    __syncthreads();
    ofs = VS > 1 ? 0 : (int64_t)sm_len[0];  // slices of one cache index its tokens themselves
    int64_t len_g = (int64_t)sm_len[1];
    if (len_g > INT32_MAX) {  // global indices are int32
      if (rank == 0 && tid == 0) atomicOr(p.err, kErrSeqLen);
      len_g = INT32_MAX;
    }
    keff = (int)min((int64_t)p.budget, len_g);
  }
  // Every block of the cluster has started (and may be written to through
  // distributed shared memory) once every thread has arrived here; each thread
  // waits on it before its first such access.
  cluster_arrive();

  // ================================================================ phase 1
  if (!worker) {
    // Stage i holds the code rows of tokens t0 + [i * kStageRows, +rows): one bulk copy
    // in a contiguous cache; in a paged cache lane 0 waits for the stage to be free and
    // arms its barrier with the stage's bytes, and the lanes copy one page piece each.
    // The lane's first kLookAhead page pieces of a stage are looked up in the block
    // table before the wait for the stage's buffer, so the table reads overlap it
    // (a bad entry is flagged once, after the stream).
    constexpr int kLookAhead = 4;
    bool bad_page = false;
    auto issue = [&](int i) {
      const int buf = i % NS;
      const int r0 = i * kStageRows, nr = min(kStageRows, seg_len - r0);
      const int ta = (int)(t0 + r0), tb = ta + nr, P = p.page_size;  // token offsets < 2^31
      const int lp0 = (int)((uint32_t)ta / (uint32_t)P) + lane, lp_end = (int)((uint32_t)(tb - 1) / (uint32_t)P);
      int64_t row[kLookAhead];
#pragma unroll
      for (int k = 0; k < kLookAhead; ++k) {
        const int lp = lp0 + 32 * k;
        row[k] = lp <= lp_end ? cache_row(p, b, kvh, max(ta, lp * P), bad_page) : 0;
      }
      if (lane == 0) {
        if (i >= NS && !mbar_wait_timed(&sm_empty[buf], (uint32_t)((i / NS) - 1) & 1u, kWaitNs))
          atomicOr(p.err, kErrTimeout);
        if (i != p.withhold) mbar_arrive_expect_tx(&sm_full[buf], (uint32_t)nr * kCodeBytes);
      }
      __syncwarp();
      if (i == p.withhold) return;  // test hook: this stage never arrives
      unsigned char* dst = ring + (size_t)buf * kStageBytes;
#pragma unroll
      for (int k = 0; k < kLookAhead; ++k) {
        const int lp = lp0 + 32 * k;
        if (lp <= lp_end) {
          const int s0 = max(ta, lp * P), s1 = min(tb, (lp + 1) * P);
          bulk_copy_g2s(dst + (size_t)(s0 - ta) * kCodeBytes, p.codes + row[k] * kCodeBytes,
                        (uint32_t)(s1 - s0) * kCodeBytes, &sm_full[buf]);
        }
      }
      for (int lp = lp0 + 32 * kLookAhead; lp <= lp_end; lp += 32) {  // pages of fewer than 8 tokens
        const int s0 = max(ta, lp * P), s1 = min(tb, (lp + 1) * P);
        bulk_copy_g2s(dst + (size_t)(s0 - ta) * kCodeBytes, p.codes + cache_row(p, b, kvh, s0, bad_page) * kCodeBytes,
                      (uint32_t)(s1 - s0) * kCodeBytes, &sm_full[buf]);
      }
    };
    if (!GENERAL || p.table == nullptr) {  // contiguous: lane 0 issues every copy alone
      if (lane == 0)
        for (int i = 0; i < nst; ++i) {
          const int buf = i % NS;
          const int r0 = i * kStageRows, nr = min(kStageRows, seg_len - r0);
          if (i >= NS && !mbar_wait_timed(&sm_empty[buf], (uint32_t)((i / NS) - 1) & 1u, kWaitNs))
            atomicOr(p.err, kErrTimeout);
          if (i == p.withhold) continue;  // test hook: this stage never arrives
          mbar_arrive_expect_tx(&sm_full[buf], (uint32_t)nr * kCodeBytes);
          bulk_copy_g2s(ring + (size_t)buf * kStageBytes, p.codes + (kv_base + t0 + r0) * kCodeBytes,
                        (uint32_t)nr * kCodeBytes, &sm_full[buf]);
        }
    } else {
      for (int i = 0; i < nst; ++i) issue(i);
      if (bad_page) atomicOr(p.err, kErrTable);
    }
    __syncwarp();
    cluster_wait();
  } else {
    if (!ATTEND_ONLY && warp < G && keff > 0) {
      const uint32_t w = encode128_warp(p.q + ((int64_t)b * p.Hq + kvh * G + warp) * kDim, lane);
      if (lane < kCodeWords) {
        sm_q[warp * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + lane] = w;
        sm_qc[warp * 2 * kCodeWords + kCodeWords + lane] = query_mask(w);
      }
    }
    if (warp == kWorkerWarps - 1 && apos >= 0) {  // the same encoder as adamas_encode_keys
      const int64_t arow_c = GENERAL ? cache_row(p, b, kvh, apos) : kv_base + apos;
      const int64_t nrow = (int64_t)b * p.Hkv + kvh;
      const bool rows_in = GENERAL && p.k_new != nullptr;
      const uint16_t* ksrc = rows_in ? p.k_new + nrow * kDim : (p.K != nullptr ? p.K + arow_c * kDim : nullptr);
      if (ksrc == nullptr || p.codes_w == nullptr) {  // never with the host's launches: flagged, nothing read
        if (lane == 0) atomicOr(p.err, kErrInternal);
      } else {
        const uint32_t w = encode128_warp(ksrc, lane);
        if (lane < kCodeWords) {
          sm_acode[lane] = w;
          reinterpret_cast<uint32_t*>(p.codes_w + arow_c * kCodeBytes)[lane] = w;
        }
        if (rows_in) {  // the new K row (lanes 0-15) and V row (lanes 16-31) into the cache
          const uint16_t* src = (lane < 16 ? p.k_new : p.v_new) + nrow * kDim + (lane & 15) * 8;
          uint16_t* dst = (lane < 16 ? p.K_w : p.V_w) + arow_c * kDim + (lane & 15) * 8;
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
        }
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
      if (!mbar_wait_timed(&sm_full[buf], (uint32_t)(i / NS) & 1u, kWaitNs)) atomicOr(p.err, kErrTimeout);
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
          // forced rows (sinks and the recent window) rank at 0, every other token at D + 1
          bool fr = false;
          if (forced) {
            const int64_t tg = t0 + t;
            fr = tg < p.n_sink || tg >= len_b - p.n_recent;
          }
          int dsum = 0;
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
            if constexpr (SHARED) {
              dsum += d;
            } else {
              if (forced) d = fr ? 0 : d + 1;
              if constexpr (SMEM_D) sts16(smem_addr(dist + (size_t)g * p.dstride + t), (uint16_t)d);
              else dist[(size_t)g * p.dstride + t] = (uint16_t)d;
              atomicAdd(&sm_hist[g * kHistStride + d], 1u);
            }
          }
          if constexpr (SHARED) {  // one distance row and one histogram for the kv head
            if (forced) dsum = fr ? 0 : dsum + 1;
            if constexpr (SMEM_D) sts16(smem_addr(dist + t), (uint16_t)dsum);
            else dist[t] = (uint16_t)dsum;
            atomicAdd(&sm_hist[dsum], 1u);
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
    if constexpr (SCORE_ONLY) {  // own histograms to the workspace, and into the slice's sums
      worker_sync();
      uint32_t* bh = p.blk_hist + (size_t)blockIdx.x * G * kHistStride;
      for (int i = tid; i < G * kHistStride; i += kWorkers) {
        const uint32_t v = sm_hist[i];
        bh[i] = v;
        const int g = i / kHistStride, d = i - g * kHistStride;
        if (v != 0u)
          atomicAdd(p.shard_hist + ((int64_t)vs * p.B * p.Hq + (int64_t)b * p.Hq + kvh * G + g) * kHistStride + d, v);
      }
    } else if constexpr (ATTEND_ONLY) {  // own histograms from the score half
      const uint32_t* bh = p.blk_hist + (size_t)blockIdx.x * G * kHistStride;
      for (int i = tid; i < G * kHistStride; i += kWorkers) sm_hist[i] = bh[i];
    } else if (push_hist && keff > 0) {  // own histograms into every block's table (row `rank`)
      worker_sync();
      for (int r = 0; r < C; ++r) {
        uint32_t* tab = cluster.map_shared_rank(sm_htab, r) + (size_t)rank * G * kHistStride;
        for (int i = tid; i < G * kHistStride; i += kWorkers) tab[i] = sm_hist[i];
      }
    }
  }
  if constexpr (SCORE_ONLY) return;  // no peer reads this block's shared memory in this mode
  __syncthreads();
  cluster.sync();  // every block's histograms are complete and visible to the cluster

  // ================================================================ phase 2
  if (worker && keff > 0) {
    // ---- the tail of the last 8-position group of every distance row reads as "far"
    if (tid < (SHARED ? 1 : G))
      for (int pos = seg_len; pos < ((seg_len + 7) & ~7); ++pos) {
        if constexpr (SMEM_D) sts16(smem_addr(dist + (size_t)tid * p.dstride + pos), 0xFFFFu);
        else dist[(size_t)tid * p.dstride + pos] = 0xFFFFu;
      }
    // ---- thresholds, rank bases and own prefixes of every selection (each query head,
    // or the kv head when the group shares one).  Thread tid takes bins
    // [tid * bpt, tid * bpt + bpt); per bin: the head's total H over the cluster's
    // blocks, the count P of the lower-ranked blocks and this block's own count.
    {
      // per-head selections have at most kBins + 1 bins: one per thread
      const int bpt = SHARED ? (nbins + kWorkers - 1) / kWorkers : 1;
      for (int g = 0; g < (SHARED ? 1 : G); ++g) {
        auto bin = [&](int d, long long& H, long long& P, long long& own) {
          H = P = own = 0;
          if (d >= nbins) return;
          if constexpr (ATTEND_ONLY) {
            // this slice: the blocks of the cluster; the other slices: their sums
            const uint32_t* bh = p.blk_hist + ((size_t)clus * C * G + g) * kHistStride + d;
            for (int r = 0; r < C; ++r) {
              const uint32_t v = bh[(size_t)r * G * kHistStride];
              H += v;
              if (r < rank) P += v;
            }
            const uint32_t* ha = p.hist_all + ((int64_t)b * p.Hq + (int64_t)kvh * G + g) * kHistStride + d;
            const int64_t rs = (int64_t)p.B * p.Hq * kHistStride;
            for (int r = 0; r < sworld; ++r) {
              if (r == srank) continue;
              const uint32_t v = ha[r * rs];
              H += v;
              if (r < srank) P += v;
            }
          } else {
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
          }
          own = sm_hist[g * kHistStride + d];
        };
        long long Hs = 0, Os = 0, H1 = 0, P1 = 0, O1 = 0;  // H1, P1, O1: the bin of a one-bin thread
        for (int j = 0; j < bpt; ++j) {
          long long H, P, own;
          bin(tid * bpt + j, H, P, own);
          Hs += H;
          Os += own;
          H1 = H;
          P1 = P;
          O1 = own;
        }
        // both prefixes in one scan: totals of the head in the high word, own counts in the low one
        const long long pre = worker_exclusive_scan(Hs << 32 | Os, sm_tmp);
        long long base = pre >> 32, obase = pre & 0xFFFFFFFFll;
        for (int j = 0; j < bpt; ++j) {
          const int d = tid * bpt + j;
          long long H = H1, P = P1, own = O1;
          if (bpt > 1) bin(d, H, P, own);
          if (d < nbins) {
            if (base < keff && base + H >= keff) sm_T[g] = d;
            sm_rank[g * kHistStride + d] = (uint32_t)(base + P);
            sm_lpre[g * kHistStride + d] = (uint32_t)obase;
          }
          base += H;
          obase += own;
        }
      }
    }
    worker_sync();

    const int hw = tid >> 4, hl = tid & 15;  // two half-warps per worker warp
    const int64_t it0 = t0 + ofs;  // index (in the whole sequence) of the block's first token
    const float kScoreScale = 0.08838834764831845f * 1.4426950408889634f;  // log2(e)/sqrt(128)
    // warp slices over 8-position groups of the block's distances (full scans)
    const int ngrp = (seg_len + 7) >> 3;
    const int gpw = (ngrp + kWorkerWarps - 1) / kWorkerWarps;
    const int wg0 = min(ngrp, warp * gpw), wg1 = min(ngrp, (warp + 1) * gpw);

    // kept tokens are gathered from the contiguous cache by their offset in the
    // block's segment, or -- in a paged cache -- by their cache row, looked up once
    const bool paged = GENERAL && p.table != nullptr;
    const int64_t grow0 = paged ? 0 : kv_base + t0;
    const uint32_t gmask = paged ? 0x7FFFFFFFu : kPosMask;  // prefetch of the fallback windows
    const int64_t glimit = paged ? p.n_pages * p.Hkv * p.page_size : (int64_t)seg_len;

    // Group-shared selection.  One pass over the block's summed distances (each
    // thread a run of 8-position groups, rounds in index order) marks D < T and D == T;
    // one block scan of the two counts lists every D < T token -- its sort key
    // (D << 32 | offset) at [0, n_lt) -- and every tie at n_lt + (its rank among the
    // block's ties), both in index order, so the first tie_quota ties are the kept
    // ones and go straight to their slots.  The D < T keys are then sorted (bitonic,
    // over the next power of two); a token's slot is the rank base of its distance plus
    // its place among the block's tokens of that distance.
    uint64_t* sm_keys = reinterpret_cast<uint64_t*>(ring);  // [kKeptCap] (below sm_kept)
    auto select_ordered_sorted = [&](const uint16_t* drow, uint32_t T, int n_lt, int n_eq, int tie_base,
                                     int tie_quota, int n_kept, const uint32_t* rank_g, const uint32_t* lpre_g,
                                     int32_t* idx_h) {
      const uint32_t t1x2 = (T + 1) | (T + 1) << 16;
      const int rot = lane & 7;
      int lt_base = 0, eq_base = 0;  // tokens placed by earlier rounds
      for (int r0 = 0; r0 < ngrp; r0 += kWorkers * 8) {
        const int span = min(kWorkers * 8, ngrp - r0);
        const int cnt = (span + kWorkers - 1) / kWorkers;
        const int g0 = r0 + tid * cnt;
        unsigned long long cm = 0ull;  // bit 8j + e: position (g0 + j) * 8 + e has D <= T
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          uint4 v[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int j = (h + u + rot) & 7, grp = g0 + j;
            v[u] = (j < cnt && grp < r0 + span) ? load_dist8<SMEM_D>(drow, grp) : make_uint4(~0u, ~0u, ~0u, ~0u);
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) cm |= (unsigned long long)le_bits(v[u], t1x2) << (8 * ((h + u + rot) & 7));
        }
        const int pbase = g0 * 8;
        int clt = 0, ceq = 0;
        for (unsigned long long mm = cm; mm != 0ull; mm &= mm - 1ull) {
          const uint32_t dd = load_dist1<SMEM_D>(drow, pbase + __ffsll((long long)mm) - 1);
          clt += dd < T;
          ceq += dd == T;
        }
        // a round holds at most kWorkers * 64 positions: both counts fit in 16 bits
        const uint32_t pre = worker_exclusive_scan32((uint32_t)clt << 16 | (uint32_t)ceq,
                                                     reinterpret_cast<uint32_t*>(sm_tmp));
        if (tid == kWorkers - 1) {
          sm_round[0] = (int)(pre >> 16) + clt;
          sm_round[1] = (int)(pre & 0xFFFFu) + ceq;
        }
        int at_lt = lt_base + (int)(pre >> 16), at_eq = eq_base + (int)(pre & 0xFFFFu);
        for (unsigned long long mm = cm; mm != 0ull; mm &= mm - 1ull) {
          const uint32_t pos = (uint32_t)(pbase + __ffsll((long long)mm) - 1);
          const uint32_t dd = load_dist1<SMEM_D>(drow, (int)pos);
          if (dd < T) {
            if (at_lt < n_lt) {
              sm_keys[at_lt] = (uint64_t)dd << 32 | pos;
              sm_kept[at_lt] = (int32_t)pos;
            } else {
              atomicOr(p.err, kErrInternal);  // never with consistent histograms
            }
            ++at_lt;
          } else {
            if (at_eq < tie_quota && n_lt + at_eq < n_kept) {
              sm_kept[n_lt + at_eq] = (int32_t)pos;
              idx_h[tie_base + at_eq] = (int32_t)(it0 + pos);
            }
            ++at_eq;
          }
        }
        worker_sync();  // the round's totals are visible
        lt_base += sm_round[0];
        eq_base += sm_round[1];
        worker_sync();  // every thread has them before a next round overwrites them
      }
      if (tid == 0 && (lt_base != n_lt || eq_base != n_eq)) atomicOr(p.err, kErrInternal);
      int n2 = 1;
      while (n2 < n_lt) n2 <<= 1;
      for (int i = n_lt + tid; i < n2; i += kWorkers) sm_keys[i] = ~0ull;
      worker_sync();
      for (int k = 2; k <= n2; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int i = tid; i < n2; i += kWorkers) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const uint64_t a = sm_keys[i], c = sm_keys[ixj];
              if ((a > c) == ((i & k) == 0)) {
                sm_keys[i] = c;
                sm_keys[ixj] = a;
              }
            }
          }
          worker_sync();
        }
      for (int i = tid; i < n_lt; i += kWorkers) {
        const uint64_t kk = sm_keys[i];
        const uint32_t d = (uint32_t)(kk >> 32);
        const uint32_t slot = rank_g[d] + ((uint32_t)i - lpre_g[d]);
        if (slot < (uint32_t)keff) idx_h[slot] = (int32_t)(it0 + (uint32_t)kk);
      }
      worker_sync();
    };

    for (int g = 0; g < G; ++g) {
      const int64_t hq = (int64_t)b * p.Hq + kvh * G + g;
      const int sg = SHARED ? 0 : g;  // the selection this query head attends over
      int32_t* idx_h = p.idx + (SHARED ? (int64_t)b * p.Hkv + kvh : hq) * p.budget;
      const uint16_t* drow = dist + (size_t)sg * p.dstride;
      const uint32_t* rank_g = sm_rank + sg * kHistStride;
      const uint32_t* lpre_g = sm_lpre + sg * kHistStride;
      const uint32_t* hist_g = sm_hist + sg * kHistStride;
      const uint32_t T = (uint32_t)sm_T[sg];
      const int tie_base = (int)rank_g[T];              // output slot of this block's first tie
      const int tie_quota = max(0, keff - tie_base);    // ties this block keeps (its first ones)
      const int n_lt = (int)lpre_g[T];                  // tokens of the block with D < T
      const int n_eq = (int)hist_g[T];                  // ties of the block
      const int n_kept = n_lt + min(tie_quota, n_eq);   // kept tokens, in slot order at [0, n_kept)
      const uint4 qraw = *reinterpret_cast<const uint4*>(p.q + hq * kDim + 8 * hl);

      float qf[8];
      float m_run = -INFINITY, l_run = 0.0f, o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = 0.0f;
      auto load_q = [&]() {
        qf[0] = bf16_lo(qraw.x) * kScoreScale; qf[1] = bf16_hi(qraw.x) * kScoreScale;
        qf[2] = bf16_lo(qraw.y) * kScoreScale; qf[3] = bf16_hi(qraw.y) * kScoreScale;
        qf[4] = bf16_lo(qraw.z) * kScoreScale; qf[5] = bf16_hi(qraw.z) * kScoreScale;
        qf[6] = bf16_lo(qraw.w) * kScoreScale; qf[7] = bf16_hi(qraw.w) * kScoreScale;
      };

      // paged cache: the kept offsets [0, n) become cache rows (one table lookup each)
      auto to_rows = [&](int n) {
        if (!paged) return;
        bool bad = false;
        for (int i = tid; i < n; i += kWorkers) {
          const uint32_t off = lds32(smem_addr(sm_kept + i)) & kPosMask;
          sm_kept[i] = (int32_t)cache_row(p, b, kvh, t0 + off, bad);
        }
        if (bad) atomicOr(p.err, kErrTable);
        worker_sync();
      };
      // gather of the kept tokens [0, n) of one window into the softmax state
      auto gather = [&](int n, bool prefetch) {
        for (int i = tid; prefetch && i < 4 * n; i += kWorkers) {  // every kept row on its way into L2
          const int64_t t = grow0 + (int64_t)(lds32(smem_addr(sm_kept + (i >> 2))) & gmask);
          prefetch_l2((i & 2 ? p.V : p.K) + t * kDim + (i & 1) * 64);
        }
        for (int rb = 2 * warp; rb < n; rb += kGatherBatch) {
          uint4 kr[kGatherRows], vr[kGatherRows];
          if (paged) gather_issue<true>(sm_kept, rb, n, hw, hl, p.K, p.V, grow0, glimit, kr, vr);
          else gather_issue<false>(sm_kept, rb, n, hw, hl, p.K, p.V, grow0, glimit, kr, vr);
          gather_fold(rb, n, hw, qf, kr, vr, m_run, l_run, o);
        }
      };

      if constexpr (SHARED) {
        if (g == 0) {
          select_ordered_sorted(drow, T, n_lt, n_eq, tie_base, tie_quota, n_kept, rank_g, lpre_g, idx_h);
          to_rows(n_kept);
        }
        load_q();
        gather(n_kept, false);
        worker_sync();
      } else {
      // The compact path: every token with D <= T (typically a few hundred) is listed
      // in index order, then ranked among the listed tokens of its distance; else the
      // two scans.
      const bool compact = n_lt + n_eq <= kListCap && n_kept <= kKeptCap;

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
              idx_h[slot] = (int32_t)(it0 + tpos);
              sm_kept[kp] = (int32_t)tpos;
            }
          }
          if (r0 + kWorkers < listed) {  // counts carried to the next round
            worker_sync();
            for (int dd = tid; dd < nbins; dd += kWorkers) {
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
        load_q();
        to_rows(n_kept);
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
        load_q();

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
                        if (c0 == 0) idx_h[tie_base + tie] = (int32_t)(it0 + pos);
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
                if (c0 == 0 && rank_g[d] + before < (uint32_t)keff) idx_h[rank_g[d] + before] = (int32_t)(it0 + tpos);
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
          to_rows(n_win);
          gather(n_win, true);
          worker_sync();
        }
      }
      }  // per-head selection
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
        float res = 0.0f, M = -INFINITY, L = 0.0f, O = 0.0f;
        if (keff > 0) {
          const float* tab = sm_ptab + (size_t)(g / C) * C * kPartial;
          for (int r = 0; r < C; ++r) M = fmaxf(M, tab[r * kPartial]);
          for (int r = 0; r < C; ++r) {
            const float mr = tab[r * kPartial];
            if (mr == -INFINITY) continue;  // a block that kept no token of this head
            const float wgt = exp2f(mr - M);
            L += tab[r * kPartial + 1] * wgt;
            O += tab[r * kPartial + 4 + e] * wgt;
          }
          res = O / L;
        }
        if constexpr (ATTEND_ONLY) {  // the slice's state (m = -inf, l = 0: it kept no token)
          float* dst = p.partial + ((int64_t)vs * p.B * p.Hq + hq) * kPartial;
          dst[4 + e] = O;
          if (e == 0) {
            dst[0] = M;
            dst[1] = L;
            dst[2] = 0.0f;
            dst[3] = 0.0f;
          }
        } else {
          p.out[hq * kDim + e] = res;
        }
      }
    }
    if (!ATTEND_ONLY && rank == 0)  // slots past k_eff (the sharded step's idx starts at -1): one row per query head, or one per kv head when shared
      for (int i = tid; i < (SHARED ? 1 : G) * p.budget; i += kWorkers) {
        const int g = i / p.budget, r = i - g * p.budget;
        const int64_t row = SHARED ? (int64_t)b * p.Hkv + kvh : (int64_t)b * p.Hq + kvh * G + g;
        if (r >= keff) p.idx[row * p.budget + r] = -1;
      }
  }
}

}  // namespace adamas
