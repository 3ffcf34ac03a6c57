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
// no grid-wide wait and no dependency between clusters.
//   phase 1  one warp streams the block's packed code rows into a ring of 32 KiB
//            shared-memory stages with bulk asynchronous copies (one full and one
//            empty mbarrier per stage); sixteen warps encode the G query heads of
//            the kv head, then score every row against them (exact L1, two rows
//            per thread per stage), keep the G distances of every token (shared
//            memory, or the workspace when they do not fit) and count them in one
//            385-bin histogram per query head.  When the cluster's histograms fit,
//            every block then writes its own into a table in each peer.
//   -- cluster barrier --
//   phase 2  per query head: the C histograms give the threshold T with
//            count(D < T) < k_eff <= count(D <= T) and, for every distance d, the
//            rank base = #tokens of the head with a smaller distance + #tokens
//            with distance d in lower-ranked blocks.  Every token with D < T is
//            kept; of the ties D == T this block keeps its first k_eff - base(T)
//            in index order, so ties go to the lowest indices.  A token's output
//            slot is its rank base + its rank by index among the block's tokens
//            of equal distance.  One pass over the block's distances lists every
//            token with D <= T (typically a few hundred) in index order (each
//            thread marks its own run of positions, lanes rotated so that a warp's
//            loads spread over the banks; one block scan of the counts gives each
//            thread its place in the list); a token's rank among the block's tokens
//            of its distance is then the number of listed tokens of that distance
//            before it (a warp match, per-warp counts, counts carried between
//            rounds of 512 entries).  When more than 4096 tokens have D <= T (heavy
//            ties) two scans take over: per-warp counts, then an in-order emit with
//            a warp match over 32-entry chunks for the D < T tokens.  Either way
//            the kept tokens end up in slot order, so both give the same bits.
//            The kept K/V rows are gathered into registers (each half-warp keeps
//            four K and four V rows in flight) and folded
//            into an online-softmax state per half-warp; the states become one
//            partial (m, l, o) per query head and block, which goes to the block
//            that owns the head's merge.
//   -- cluster barrier --
//   merge    each block combines the C partial states of the query heads it owns
//            (g mod C == its rank) into out; block 0 pads idx with -1.
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
constexpr int kStageRows = 2 * kWorkers;              // code rows per ring stage (two per worker)
constexpr uint32_t kStageBytes = kStageRows * kCodeBytes;  // 32 KiB
constexpr int kRowsPerThread = kStageRows / kWorkers;
constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
constexpr int kMaxCluster = 16;
constexpr int kHistStride = 388;                      // >= kBins, multiple of 4
constexpr int kPartial = 132;                         // m, l, pad, pad, o[128]
constexpr int kListCap = 4096;                        // D < T tokens listed per round / grouped tokens D <= T
constexpr int kKeptCap = 4096;                        // kept tokens per gather window
constexpr int kGatherRows = 4;                        // K/V rows in flight per half-warp
constexpr int kScanBatch = 4;                         // 32-group iterations of a distance scan loaded together
constexpr int kGatherBatch = 2 * kWorkerWarps * kGatherRows;  // rows per gather batch of the block
constexpr int kPushHistMax = 8;                       // C * G up to which histograms are pushed to peers
constexpr uint32_t kPosMask = (1u << 23) - 1u;        // token offset within a block (list entries: d << 23 | t)
constexpr uint32_t kWaitLimit = 1u << 20;             // mbarrier polls (about a second)
constexpr uint64_t kWaitNs = 1000000000ull;          // time bound of a wait of the step with options

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
  uint8_t* codes_w;     // writable codes when appending (the same array as codes), else null
  const int32_t* append_pos;  // [B] position whose key is encoded before scoring (null: none)
  const uint16_t* k_new;  // [B][Hkv][128] appended key rows written into K by the launch (null: read from K)
  const uint16_t* v_new;  // [B][Hkv][128] appended value rows written into V (with k_new)
  uint16_t* K_w;          // writable K and V (the same arrays as K, V) when k_new is given
  uint16_t* V_w;
  const int32_t* table;   // [B][max_pages] physical page of each logical page (null: contiguous cache)
  int64_t n_pages;        // physical pages (paged cache)
  int page_size, max_pages;
  int n_sink, n_recent;   // forced rows: the first n_sink and the last n_recent tokens of each sequence
  int withhold;           // test hook: the stage whose copy is never issued (-1: none)
  // sequence-sharded step: the cache holds one contiguous slice of every sequence
  uint32_t* shard_hist;       // score: [B][Hq][kHistStride] this slice's histograms (added into, zeroed first)
  const uint32_t* hist_all;   // attend: [world][B][Hq][kHistStride] the histograms of every slice, in order
  uint32_t* blk_hist;         // [grid][G][kHistStride] each block's own histograms (workspace)
  float* partial;             // attend: [B][Hq][kPartial] this slice's softmax state (m, l, -, -, o[128])
  int shard_rank, shard_world;
  int vslices;                // sharded modes on one GPU: slices per (b, kv head) in this launch (1: none)
  int B, Hq, Hkv;
  int64_t Nmax;           // tokens per sequence the cache can hold (paged: max_pages * page_size)
  int budget;
  int cluster;          // blocks per (b, kv head)
  int nstages;          // ring stages, kMinStages..kMaxStages
  int dstride;          // distances per query head and block (>= any block's tokens, multiple of 64)
};

// Shared-memory carve-up (bytes), shared with the host.
//   head:  q codes [G][8] | q words + masks [G][16] | own histograms [G][kHistStride]
//          | rank bases [G][kHistStride] | own exclusive prefix [G][kHistStride]
//          | histogram table [C][G][kHistStride] (when C*G <= kPushHistMax)
//          | partial-state table [ceil(G/C)*C][kPartial]
//   ring:  nstages x 32 KiB; in phase 2: per-warp chunk counts [kWorkerWarps][kHistStride]
//          (later the half-warp softmax states), carried counts / group cursors
//          [kHistStride], D < T tokens or grouped candidates [kListCap], kept tokens [kKeptCap]
//   dist:  [G][dstride] u16 when kept in shared memory
struct DecodeSmem {
  static __host__ __device__ inline size_t align128(size_t x) { return (x + 127) / 128 * 128; }
  static __host__ __device__ inline bool push_hist(int G, int C) { return G * C <= kPushHistMax; }
  static __host__ __device__ inline int owned(int G, int C) { return (G + C - 1) / C; }
  static __host__ __device__ inline size_t qcodes(int G) { return align128((size_t)G * kCodeWords * 4); }
  static __host__ __device__ inline size_t qconst(int G) { return align128((size_t)G * 2 * kCodeWords * 4); }
  static __host__ __device__ inline size_t hist(int G) { return align128((size_t)G * kHistStride * 4); }
  static __host__ __device__ inline size_t htab(int G, int C) {
    return push_hist(G, C) ? align128((size_t)C * G * kHistStride * 4) : 0;
  }
  static __host__ __device__ inline size_t ptab(int G, int C) {
    return align128((size_t)owned(G, C) * C * kPartial * 4);
  }
  static __host__ __device__ inline size_t head(int G, int C) {
    return qcodes(G) + qconst(G) + 3 * hist(G) + htab(G, C) + ptab(G, C);
  }
  static __host__ __device__ inline size_t ring(int nstages) { return (size_t)nstages * kStageBytes; }
  static constexpr __host__ __device__ size_t cnt() { return (size_t)kWorkerWarps * kHistStride * 4; }
  static constexpr __host__ __device__ size_t carry() { return (size_t)kHistStride * 4; }
  static constexpr __host__ __device__ size_t state() { return (size_t)2 * kWorkerWarps * kPartial * 4; }
  static __host__ __device__ inline size_t dist(int G, int dstride, bool in_smem) {
    return in_smem ? align128((size_t)G * dstride * 2) : 0;
  }
  static __host__ __device__ inline size_t total(int G, int C, int nstages, int dstride, bool in_smem) {
    return head(G, C) + ring(nstages) + dist(G, dstride, in_smem);
  }
};
static_assert(DecodeSmem::cnt() >= DecodeSmem::state(), "softmax states overlay the chunk counts");
static_assert(DecodeSmem::cnt() + DecodeSmem::carry() + (kListCap + kKeptCap) * 4 <= kMinStages * kStageBytes,
              "phase-2 arrays fit in the smallest ring");
static_assert(kKeptCap * 8 <= DecodeSmem::cnt() + DecodeSmem::carry() + kListCap * 4,
              "the sort keys of the group-shared selection lie below the kept list");

// ------------------------------------------------------------------ block helpers
// Barrier of the worker warps (the copy warp does not take part).
__device__ __forceinline__ void worker_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kWorkers) : "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Exclusive scan of one int64 per worker thread; returns the prefix.  Uses sm_tmp[kWorkerWarps].
__device__ __forceinline__ long long worker_exclusive_scan(long long v, long long* sm_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o *= 2) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm_tmp[warp] = x;
  worker_sync();
  long long before = 0;
#pragma unroll
  for (int w = 0; w < kWorkerWarps; ++w) before += w < warp ? sm_tmp[w] : 0;
  worker_sync();
  return before + x - v;
}

// Exclusive scan of one uint32 per worker thread; returns the prefix.  Uses
// sm_tmp[2 * kWorkerWarps]: warp 0 scans the warp totals, each thread reads one word.
__device__ __forceinline__ uint32_t worker_exclusive_scan32(uint32_t v, uint32_t* sm_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o *= 2) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm_tmp[warp] = x;
  worker_sync();
  if (warp == 0) {
    const uint32_t t = lane < kWorkerWarps ? sm_tmp[lane] : 0u;
    uint32_t u = t;
#pragma unroll
    for (int o = 1; o < kWorkerWarps; o *= 2) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) u += y;
    }
    if (lane < kWorkerWarps) sm_tmp[kWorkerWarps + lane] = u - t;
  }
  worker_sync();
  return sm_tmp[kWorkerWarps + warp] + x - v;
}

// Eight consecutive distances 8*grp .. 8*grp+7 as four words of u16 pairs (element
// 2j in the low half of word j); SMEM: the row is in shared memory.
template <bool SMEM>
__device__ __forceinline__ uint4 load_dist8(const uint16_t* drow, int grp) {
  if constexpr (SMEM) return lds128(smem_addr(drow + (size_t)grp * 8));
  else return *reinterpret_cast<const uint4*>(drow + (size_t)grp * 8);
}

template <bool SMEM>
__device__ __forceinline__ uint32_t load_dist1(const uint16_t* drow, int pos) {
  if constexpr (SMEM) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_addr(drow + pos)) : "memory");
    return v;
  } else {
    return drow[pos];
  }
}

constexpr uint32_t kHalfTops = 0x80008000u;

// Whether any of the eight distances is <= T (t1x2 = (T+1) in both halves).  With
// distances below 2^15 (0xFFFF pads a row), (x | 0x8000) - (T+1) keeps bit 15 of its
// half exactly when x > T, and no half borrows from the other.
__device__ __forceinline__ bool any_le(const uint4 v, uint32_t t1x2) {
  const uint32_t a = ((v.x | kHalfTops) - t1x2) & ((v.y | kHalfTops) - t1x2) & ((v.z | kHalfTops) - t1x2) &
                     ((v.w | kHalfTops) - t1x2);
  return (a & kHalfTops) != kHalfTops;
}

// Bit e set when distance e of the eight is <= T; t1x2 = T+1 in both halves.
__device__ __forceinline__ uint32_t le_bits(const uint4 v, uint32_t t1x2) {
  const uint32_t l0 = ~((v.x | kHalfTops) - t1x2) & kHalfTops;  // bit 15: low half <= T, bit 31: high half
  const uint32_t l1 = ~((v.y | kHalfTops) - t1x2) & kHalfTops;
  const uint32_t l2 = ~((v.z | kHalfTops) - t1x2) & kHalfTops;
  const uint32_t l3 = ~((v.w | kHalfTops) - t1x2) & kHalfTops;
  const uint32_t m = (l0 >> 15) | (l1 >> 13) | (l2 >> 11) | (l3 >> 9);  // low halves at 0,2,4,6, high at 16..22
  return (m | (m >> 15)) & 0xFFu;
}

// Bit e of lt (eq) set when distance e of the eight is < T (== T); tx2 = T in both
// halves, t1x2 = T+1 in both halves.
__device__ __forceinline__ void cand_bits(const uint4 v, uint32_t tx2, uint32_t t1x2, uint32_t& lt, uint32_t& eq) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  lt = 0u;
  eq = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t ge = (w[j] | kHalfTops) - tx2;   // tops: x >= T
    const uint32_t gt = (w[j] | kHalfTops) - t1x2;  // tops: x > T
    const uint32_t l = ~ge & kHalfTops, e = ge & ~gt & kHalfTops;
    lt |= ((l >> 15) & 1u) << (2 * j) | (l >> 31) << (2 * j + 1);
    eq |= ((e >> 15) & 1u) << (2 * j) | (e >> 31) << (2 * j + 1);
  }
}

// A batch of kGatherRows K/V rows (16 bytes of each per lane of a half-warp) folded
// into the half-warp's online-softmax state: the scores first (reduced with
// shuffles inside the half-warp; every lane of the warp takes part), then one
// rescale for the batch.  valid[j] is uniform within a half-warp.
__device__ __forceinline__ void softmax_fold(const float (&qf)[8], const uint4 (&kr)[kGatherRows],
                                             const uint4 (&vr)[kGatherRows], const bool (&valid)[kGatherRows],
                                             float& m_run, float& l_run, float (&o)[8]) {
  float sc[kGatherRows];
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j) {
    const uint4 k = kr[j];
    sc[j] = qf[0] * bf16_lo(k.x) + qf[1] * bf16_hi(k.x) + qf[2] * bf16_lo(k.y) + qf[3] * bf16_hi(k.y) +
            qf[4] * bf16_lo(k.z) + qf[5] * bf16_hi(k.z) + qf[6] * bf16_lo(k.w) + qf[7] * bf16_hi(k.w);
  }
#pragma unroll
  for (int off = 8; off > 0; off /= 2)
#pragma unroll
    for (int j = 0; j < kGatherRows; ++j) sc[j] += __shfl_xor_sync(0xffffffffu, sc[j], off);
  bool any = false;
  float mx = m_run;
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j)
    if (valid[j]) {
      any = true;
      mx = fmaxf(mx, sc[j]);
    }
  if (!any) return;
  const float corr = exp2f(m_run - mx);  // 0 while the state is empty (m_run = -inf)
  l_run *= corr;
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] *= corr;
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j)
    if (valid[j]) {
      const float pr = exp2f(sc[j] - mx);
      l_run += pr;
      const uint4 v = vr[j];
      o[0] += pr * bf16_lo(v.x); o[1] += pr * bf16_hi(v.x); o[2] += pr * bf16_lo(v.y); o[3] += pr * bf16_hi(v.y);
      o[4] += pr * bf16_lo(v.z); o[5] += pr * bf16_hi(v.z); o[6] += pr * bf16_lo(v.w); o[7] += pr * bf16_hi(v.w);
    }
  m_run = mx;
}

// K/V rows of kept entries rb + 32 j + (half-warp parity), j < kGatherRows, into
// registers.  Entry e names cache row row0 + (e & mask); an entry at or past `limit`
// (never with consistent counts, which the selection checks) reads row row0 instead,
// so every access stays in bounds.
template <bool PAGED>
__device__ __forceinline__ void gather_issue(const int32_t* kept, int rb, int n, int hw, int hl, const uint16_t* K,
                                             const uint16_t* V, int64_t row0, int64_t limit,
                                             uint4 (&kr)[kGatherRows], uint4 (&vr)[kGatherRows]) {
  constexpr uint32_t mask = PAGED ? 0x7FFFFFFFu : kPosMask;  // cache rows, or offsets in the block's segment
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j) {
    const int row = rb + 2 * kWorkerWarps * j + (hw & 1);
    kr[j] = make_uint4(0u, 0u, 0u, 0u);
    vr[j] = kr[j];
    if (row < n) {
      uint32_t off = lds32(smem_addr(kept + row)) & mask;
      off = (PAGED ? (int64_t)off < limit : off < (uint32_t)limit) ? off : 0u;  // clamp, no branch
      const int64_t t = row0 + off;
      kr[j] = __ldcg(reinterpret_cast<const uint4*>(K + t * kDim) + hl);
      vr[j] = __ldcg(reinterpret_cast<const uint4*>(V + t * kDim) + hl);
    }
  }
}

// The plain step's gatherer: K/V rows of kept entries rb + 32 j + (half-warp parity),
// j < kGatherRows, into registers; `kept` holds token offsets within the block.
__device__ __forceinline__ void gather_issue_plain(const int32_t* kept, int rb, int n, int hw, int hl, const uint16_t* K,
                                             const uint16_t* V, int64_t row0, uint4 (&kr)[kGatherRows],
                                             uint4 (&vr)[kGatherRows]) {
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j) {
    const int row = rb + 2 * kWorkerWarps * j + (hw & 1);
    kr[j] = make_uint4(0u, 0u, 0u, 0u);
    vr[j] = kr[j];
    if (row < n) {
      const int64_t t = row0 + (int64_t)lds32(smem_addr(kept + row));
      kr[j] = __ldcg(reinterpret_cast<const uint4*>(K + t * kDim) + hl);
      vr[j] = __ldcg(reinterpret_cast<const uint4*>(V + t * kDim) + hl);
    }
  }
}

__device__ __forceinline__ void gather_fold(int rb, int n, int hw, const float (&qf)[8], const uint4 (&kr)[kGatherRows],
                                            const uint4 (&vr)[kGatherRows], float& m_run, float& l_run,
                                            float (&o)[8]) {
  bool valid[kGatherRows];
#pragma unroll
  for (int j = 0; j < kGatherRows; ++j) valid[j] = rb + 2 * kWorkerWarps * j + (hw & 1) < n;
  softmax_fold(qf, kr, vr, valid, m_run, l_run, o);
}

// Cache row of token t of (b, kv head): [B][Hkv][Nmax] when contiguous; through
// the block table otherwise, pages laid out [page][Hkv][page_size].  An entry
// outside [0, n_pages) reads page 0 (accesses stay in bounds) and sets `bad`; the
// caller flags it.  No branch depends on the table entry, so a warp does not stall
// on the table read until it uses the row.
__device__ __forceinline__ int64_t cache_row(const DecodeParams& p, int b, int kvh, int64_t t, bool& bad) {
  if (p.table == nullptr) return ((int64_t)b * p.Hkv + kvh) * p.Nmax + t;
  const int lp = (int)((uint32_t)t / (uint32_t)p.page_size);  // t < 2^31
  const int off = (int)t - lp * p.page_size;
  const int64_t page = p.table[(int64_t)b * p.max_pages + lp];
  const bool ok = page >= 0 && page < p.n_pages;
  bad |= !ok;
  return ((ok ? page : 0) * p.Hkv + kvh) * p.page_size + off;
}

__device__ __forceinline__ int64_t cache_row(const DecodeParams& p, int b, int kvh, int64_t t) {
  bool bad = false;
  const int64_t r = cache_row(p, b, kvh, t, bad);
  if (bad) atomicOr(p.err, kErrTable);
  return r;
}

}  // namespace adamas
