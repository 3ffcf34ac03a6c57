// C ABI of the ADAMAS sparse decode library (declared in include/adamas.h):
// argument checks, workspace layout, and the launches of the sm_100a kernels.
//
// Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
// §2.1 Hadamard rotation, §2.2 dynamic 2-bit bucketing, §3.1 packed code cache,
// §2.3 Manhattan-distance scoring, §5.2 token budget.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/adamas.h"
#include "common.cuh"
#include "decode_ext.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

// ------------------------------------------------------------------ key encoder
// Prefill: one vector per thread.  Work is handed out in tiles of 32 consecutive
// positions of one (b, kv head), one tile per warp at a time: the warp copies the
// next tile into its other shared-memory buffer with coalesced 16-byte cp.async
// (two rows per instruction) while it encodes the current one, each lane reading
// its own row.  Rows are padded to 272 B, so the 16-byte reads of a quarter-warp
// fall into distinct banks.  The loop has no block-wide barrier.
constexpr int kEncWarps = 4;
constexpr int kEncThreads = 32 * kEncWarps;
constexpr int kEncRowBytes = 272;
constexpr int kEncWarpStage = 32 * kEncRowBytes;
constexpr size_t kEncSmem = (size_t)2 * kEncWarps * kEncWarpStage;  // 69,632 B
constexpr int kEncBlocksPerSm = 3;

__global__ void __launch_bounds__(kEncThreads, kEncBlocksPerSm)
    encode_keys_kernel(const uint16_t* __restrict__ K, uint8_t* __restrict__ codes,
                       const int32_t* __restrict__ pos_begin, int count, int Hkv, int64_t Nmax, int tiles_per_head,
                       int heads) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char* wbuf = smem + (size_t)warp * 2 * kEncWarpStage;

  // The warp's tiles are T = first + k * nwarps; T = hk * tiles_per_head + tin.  The
  // walk is kept incremental (one division per warp) so that the per-tile cost stays
  // a few integer operations.
  const int nwarps = gridDim.x * kEncWarps;
  const int first = blockIdx.x * kEncWarps + warp;
  int hk = first / tiles_per_head, tin = first - hk * tiles_per_head;
  const int dhk = nwarps / tiles_per_head, dtin = nwarps - dhk * tiles_per_head;

  // the tile (hk, tin): positions p0 + [0, 32) of head hk, rows [lo, hi) of it valid
  struct Tile {
    const uint16_t* src;  // key row of offset 0
    uint8_t* dst;         // code row of offset 0
    int lo, hi;
  };
  auto tile_of = [&](int h, int t) {
    const int off0 = t * 32;
    const int64_t p0 = (pos_begin ? (int64_t)pos_begin[(unsigned)h / (unsigned)Hkv] : 0) + off0;
    const int64_t row0 = (int64_t)h * Nmax + p0;
    const int64_t lo = p0 < 0 ? -p0 : 0;
    int64_t hi = count - off0 < 32 ? count - off0 : 32;
    if (Nmax - p0 < hi) hi = Nmax - p0;
    Tile r;
    r.src = K + row0 * kDim;
    r.dst = codes + row0 * kCodeBytes;
    r.lo = (int)(lo < 32 ? lo : 32);
    r.hi = (int)(hi < r.lo ? r.lo : hi);
    return r;
  };
  auto issue = [&](const Tile& t, int stage) {
    // lane l copies 16-byte chunk (l mod 16) of rows 2 s + l / 16
    unsigned char* dst = wbuf + (size_t)stage * kEncWarpStage + (lane >> 4) * kEncRowBytes + (lane & 15) * 16;
    const uint16_t* src = t.src + (lane >> 4) * kDim + (lane & 15) * 8;
    if (t.lo == 0 && t.hi == 32) {  // a whole tile: constant offsets, no checks
#pragma unroll
      for (int s = 0; s < 16; ++s) cp_async16(dst + 2 * s * kEncRowBytes, src + 2 * s * kDim);
    } else {
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const int r = 2 * s + (lane >> 4);
        if (r >= t.lo && r < t.hi) cp_async16(dst + 2 * s * kEncRowBytes, src + 2 * s * kDim);
      }
    }
    cp_async_commit();
  };

  bool more = hk < heads;
  Tile cur = tile_of(more ? hk : 0, more ? tin : 0);
  if (more) issue(cur, 0);
  else cp_async_commit();
  for (int k = 0; more; ++k) {
    tin += dtin;
    hk += dhk;
    if (tin >= tiles_per_head) {
      tin -= tiles_per_head;
      ++hk;
    }
    more = hk < heads;
    Tile nxt = cur;
    if (more) {
      nxt = tile_of(hk, tin);
      issue(nxt, (k + 1) & 1);
    } else {
      cp_async_commit();
    }
    cp_async_wait<1>();  // this lane's copies of the current tile have landed
    __syncwarp();        // ... and every other lane's
    const bool ok = lane >= cur.lo && lane < cur.hi;
    uint64_t P[kDim / 2];
    const unsigned char* row = wbuf + (size_t)(k & 1) * kEncWarpStage + lane * kEncRowBytes;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 v = ok ? *reinterpret_cast<const uint4*>(row + c * 16) : make_uint4(0u, 0u, 0u, 0u);
      P[4 * c + 0] = rotate_pair_first(v.x);
      P[4 * c + 1] = rotate_pair_first(v.y);
      P[4 * c + 2] = rotate_pair_first(v.z);
      P[4 * c + 3] = rotate_pair_first(v.w);
    }
    __syncwarp();  // every lane has read its row before the buffer is refilled
    if (ok) {
      rotate_pairs_rest(P);
      uint32_t w[kCodeWords];
      bucket_pack_pairs(P, w);
      uint4* dst = reinterpret_cast<uint4*>(cur.dst + lane * kCodeBytes);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    cur = nxt;
  }
  cp_async_wait<0>();
}

// Small encodes (appending a few tokens): one warp per vector, so a call costs
// one warp-level rotation instead of a thread walking 896 dependent adds.
constexpr int kEncWarpThreads = 256;
constexpr int64_t kEncWarpMaxVectors = 8192;

__global__ void __launch_bounds__(kEncWarpThreads) encode_keys_warp_kernel(const uint16_t* __restrict__ K,
                                                                           uint8_t* __restrict__ codes,
                                                                           const int32_t* __restrict__ pos_begin,
                                                                           int count, int Hkv, int64_t Nmax,
                                                                           int64_t nvec) {
  const int lane = threadIdx.x & 31;
  const int64_t v = (int64_t)blockIdx.x * (kEncWarpThreads / 32) + (threadIdx.x >> 5);
  if (v >= nvec) return;  // whole warp leaves together
  const int64_t hk = v / count, r = v - hk * count;
  const int b = (int)(hk / Hkv);
  const int64_t pos = (pos_begin ? (int64_t)pos_begin[b] : 0) + r;
  if (pos < 0 || pos >= Nmax) return;  // whole warp leaves together
  const int64_t row = hk * Nmax + pos;
  const uint32_t w = encode128_warp(K + row * kDim, lane);
  if (lane < kCodeWords) reinterpret_cast<uint32_t*>(codes + row * kCodeBytes)[lane] = w;
}

// ------------------------------------------------------------------ distance dump (test entry point)
constexpr int kScoreThreads = 256;
constexpr int kScoreUnroll = 4;

template <int G>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const uint16_t* __restrict__ q,
                                                              const uint8_t* __restrict__ codes,
                                                              const int32_t* __restrict__ seq_lens, int Hq,
                                                              int Hkv, int64_t Nmax, uint16_t* __restrict__ dist) {
  __shared__ uint32_t sq[G * kCodeWords];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hk = blockIdx.y, b = hk / Hkv, kvh = hk - b * Hkv;
  if (warp < G) {
    const uint32_t w = encode128_warp(q + ((int64_t)b * Hq + kvh * G + warp) * kDim, lane);
    if (lane < kCodeWords) sq[warp * kCodeWords + lane] = w;
  }
  __syncthreads();
  int64_t len = seq_lens[b];
  len = len < 0 ? 0 : (len > Nmax ? Nmax : len);
  uint32_t qw[G][kCodeWords], qm[G][kCodeWords];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w = 0; w < kCodeWords; ++w) {
      qw[g][w] = sq[g * kCodeWords + w];
      qm[g][w] = query_mask(qw[g][w]);
    }
  const int64_t first = (int64_t)blockIdx.x * kScoreThreads * kScoreUnroll;
#pragma unroll
  for (int j = 0; j < kScoreUnroll; ++j) {
    const int64_t t = first + (int64_t)j * kScoreThreads + tid;
    if (t >= Nmax) break;
    uint32_t kc[kCodeWords], k1[kCodeWords];
    if (t < len) {
      ld_stream_v8(codes + ((int64_t)hk * Nmax + t) * kCodeBytes, kc);
      key_shift(kc, k1);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint16_t d = t < len ? (uint16_t)l1_distance(kc, k1, qw[g], qm[g]) : (uint16_t)0xFFFF;
      dist[((int64_t)b * Hq + kvh * G + g) * Nmax + t] = d;
    }
  }
}

// ------------------------------------------------------------------ merge of softmax states
// Combines n partial softmax states of every (b, query head) -- the slices of a
// sharded sequence -- into the attention output.  A state is (m, l, -, -, o[128]):
// m the largest scaled score of its kept tokens in log2 units (score / sqrt(128) *
// log2 e), l the sum of 2^(s - m), o the 2^(s - m)-weighted sum of the V rows; a
// state with m = -inf kept no token.  out = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r
// with M = max_r m_r (0 when no state kept a token).  One block per (b, query head),
// one thread per output dimension.
__global__ void __launch_bounds__(kDim) merge_partials_kernel(const float* __restrict__ part, int n, int64_t rows,
                                                              float* __restrict__ out) {
  const int64_t row = blockIdx.x;
  const int e = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < n; ++r) M = fmaxf(M, part[((int64_t)r * rows + row) * kPartial]);
  float L = 0.0f, O = 0.0f;
  if (M != -INFINITY)
    for (int r = 0; r < n; ++r) {
      const float* st = part + ((int64_t)r * rows + row) * kPartial;
      if (st[0] == -INFINITY) continue;
      const float w = exp2f(st[0] - M);
      L += st[1] * w;
      O += st[4 + e] * w;
    }
  out[row * kDim + e] = M == -INFINITY ? 0.0f : O / L;
}

// ------------------------------------------------------------------ host side
constexpr int kMaxDevices = 64;
constexpr int kMinTokensPerBlock = 2048;  // fewer tokens per block than this only when the context is short
constexpr int kOccCache = 64;

struct OccEntry {
  const void* fn;
  int cluster;
  size_t smem;
  int clusters;  // cudaOccupancyMaxActiveClusters
};

struct Plan;

struct DeviceInfo {
  int sms = 0;
  size_t smem_optin = 0;
  bool attrs_set[5][2][kMaxGroup + 1] = {};  // [mode][smem_d][G]
  OccEntry occ[kOccCache] = {};
  int n_occ = 0;
  int enc_blocks_per_sm = 0;  // resident prefill-encoder blocks per SM (0: not yet set up)
};

static std::mutex g_mutex;
static DeviceInfo g_devices[kMaxDevices];
static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Record a failed CUDA call for adamas_last_error_string and map it to a status.
static int cuda_fail(cudaError_t e) {
  g_last_cuda_error = e;
  return ADAMAS_ERR_CUDA;
}

// Shared memory a block can use beyond the decode kernel's static shared memory.
constexpr size_t kStaticSmemReserve = 2048;

static int device_info(DeviceInfo** out, int* dev_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return ADAMAS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (d.sms == 0) {
    int sms = 0, optin = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return cuda_fail(e);
    d.smem_optin = (size_t)optin > kStaticSmemReserve ? (size_t)optin - kStaticSmemReserve : 0;
    d.sms = sms;
  }
  *out = &d;
  if (dev_out) *dev_out = dev;
  return ADAMAS_OK;
}

// One-time attributes of a decode kernel instance: the opt-in dynamic shared
// memory and clusters of more than 8 blocks.
static int kernel_attrs(DeviceInfo& dev, const void* fn, int G, bool smem_d, int mode) {
  std::lock_guard<std::mutex> lock(g_mutex);
  bool& done = dev.attrs_set[mode][smem_d ? 1 : 0][G];
  if (done) return ADAMAS_OK;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dev.smem_optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return cuda_fail(e);
  done = true;
  return ADAMAS_OK;
}

// One-time set-up of the prefill encoder on a device: its dynamic shared memory
// and how many of its blocks an SM holds (the persistent grid's size).
static int encoder_attrs(DeviceInfo& dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (dev.enc_blocks_per_sm > 0) return ADAMAS_OK;
  const void* fn = reinterpret_cast<const void*>(&encode_keys_kernel);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kEncSmem);
  int n = 0;
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kEncThreads, kEncSmem);
  if (e != cudaSuccess) return cuda_fail(e);
  dev.enc_blocks_per_sm = n < 1 ? 1 : n;
  return ADAMAS_OK;
}

// How many clusters of `cluster` blocks with `smem` bytes each can be resident at
// once (cached per device).
static int active_clusters(DeviceInfo& dev, const void* fn, int cluster, size_t smem, int* n) {
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int i = 0; i < dev.n_occ; ++i)
      if (dev.occ[i].fn == fn && dev.occ[i].cluster == cluster && dev.occ[i].smem == smem) {
        *n = dev.occ[i].clusters;
        return ADAMAS_OK;
      }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // an unsupported cluster size is not sticky; treat it as 0
    clusters = 0;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (dev.n_occ < kOccCache) dev.occ[dev.n_occ++] = OccEntry{fn, cluster, smem, clusters};
  *n = clusters;
  return ADAMAS_OK;
}

// Decode kernel instances live in one translation unit per group size.
#define ADAMAS_DECL_G(N)                                                                            \
  const void* decode_fn_g##N(bool smem_d, int mode);                                             \
  cudaError_t decode_launch_g##N(const cudaLaunchConfig_t* cfg, const DecodeParams& prm, bool smem_d, \
                                 int mode);
ADAMAS_DECL_G(1) ADAMAS_DECL_G(2) ADAMAS_DECL_G(3) ADAMAS_DECL_G(4)
ADAMAS_DECL_G(5) ADAMAS_DECL_G(6) ADAMAS_DECL_G(7) ADAMAS_DECL_G(8)
#undef ADAMAS_DECL_G

static const void* decode_fn_for(int G, bool smem_d, int mode) {
  switch (G) {
    case 1: return decode_fn_g1(smem_d, mode);
    case 2: return decode_fn_g2(smem_d, mode);
    case 3: return decode_fn_g3(smem_d, mode);
    case 4: return decode_fn_g4(smem_d, mode);
    case 5: return decode_fn_g5(smem_d, mode);
    case 6: return decode_fn_g6(smem_d, mode);
    case 7: return decode_fn_g7(smem_d, mode);
    case 8: return decode_fn_g8(smem_d, mode);
    default: return nullptr;
  }
}

static cudaError_t decode_launch_for(int G, const cudaLaunchConfig_t* cfg, const DecodeParams& prm, bool smem_d,
                                     int mode) {
  switch (G) {
    case 1: return decode_launch_g1(cfg, prm, smem_d, mode);
    case 2: return decode_launch_g2(cfg, prm, smem_d, mode);
    case 3: return decode_launch_g3(cfg, prm, smem_d, mode);
    case 4: return decode_launch_g4(cfg, prm, smem_d, mode);
    case 5: return decode_launch_g5(cfg, prm, smem_d, mode);
    case 6: return decode_launch_g6(cfg, prm, smem_d, mode);
    case 7: return decode_launch_g7(cfg, prm, smem_d, mode);
    case 8: return decode_launch_g8(cfg, prm, smem_d, mode);
    default: return cudaErrorInvalidValue;
  }
}

// Launch plan and workspace layout of one decode step.
struct Plan {
  int G = 1;
  int cluster = 1;   // blocks per (b, kv head)
  int grid = 0;
  int nstages = kMaxStages;
  int dstride = 64;
  bool smem_d = true;
  size_t smem = 0;
  size_t ctrl = 0, dspill = 0, bhist = 0, total = 0;  // workspace offsets / size
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static int check_shape(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nmax < 0 || budget < 0) return ADAMAS_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ADAMAS_ERR_INVALID_ARG;
  if (d != kDim) return ADAMAS_ERR_UNSUPPORTED;
  if (Hq / Hkv > kMaxGroup || B > kMaxBatch || Nmax > INT32_MAX) return ADAMAS_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv > 65535) return ADAMAS_ERR_UNSUPPORTED;
  return ADAMAS_OK;
}

// Shared-memory layout for `cluster` blocks per head: distances in shared memory
// with as many ring stages as fit, else (or when `global_d`) in the workspace with
// a full ring.
static bool layout_for(int G, int64_t Nmax, int cluster, size_t optin, bool global_d, Plan* P) {
  const int64_t seg_cap = (Nmax + cluster - 1) / cluster;  // tokens of any block
  if (seg_cap >= (int64_t(1) << 23)) return false;          // token offsets are packed in 23 bits
  P->cluster = cluster;
  P->dstride = (int)((seg_cap < 1 ? 1 : seg_cap) + 63) / 64 * 64;
  bool found = false;
  for (int pass = global_d ? 1 : 0; pass < 2 && !found; ++pass) {
    const bool in_smem = pass == 0;
    for (int ns = kMaxStages; ns >= kMinStages && !found; --ns) {
      const size_t s = DecodeSmem::total(G, cluster, ns, P->dstride, in_smem);
      if (s <= optin) {
        P->smem_d = in_smem;
        P->nstages = ns;
        P->smem = s;
        found = true;
      }
    }
  }
  if (!found) return false;
  return true;
}

// Cluster size: the largest that keeps every cluster resident at once (one
// wave), at most one block per SM in total, and at least kMinTokensPerBlock
// tokens per block; 1 when even single blocks need several waves.
static int make_plan_uncached(int B, int Hq, int Hkv, int64_t Nmax, int mode, DeviceInfo& dev, Plan* P) {
  const int G = Hq / Hkv;
  const bool sharded = mode == kModeShardScore || mode == kModeShardAttend;
  const int heads = B * Hkv;
  P->G = G;
  int want = heads > 0 ? dev.sms / heads : 1;
  const int64_t by_len = (Nmax + kMinTokensPerBlock - 1) / kMinTokensPerBlock;
  if ((int64_t)want > by_len) want = (int)by_len;
  if (want > kMaxCluster) want = kMaxCluster;
  if (want < 1) want = 1;
  bool found = false;
  for (int c = want; c >= 1 && !found; --c) {
    Plan t = *P;
    if (!layout_for(G, Nmax, c, dev.smem_optin, sharded, &t)) continue;
    const void* fn = decode_fn_for(G, t.smem_d, mode);
    int rc = kernel_attrs(dev, fn, G, t.smem_d, mode);
    if (rc != ADAMAS_OK) return rc;
    int n = 0;
    if ((rc = active_clusters(dev, fn, c, t.smem, &n)) != ADAMAS_OK) return rc;
    if (n >= 1 && (n >= heads || c == 1)) {
      *P = t;
      found = true;
    }
  }
  if (!found) return ADAMAS_ERR_UNSUPPORTED;
  P->grid = heads * P->cluster;
  size_t off = 0;
  P->ctrl = off;   off += align256(64 * sizeof(uint32_t));
  P->dspill = off;
  off += P->smem_d ? 0 : align256((size_t)P->grid * G * P->dstride * sizeof(uint16_t));
  P->bhist = off;  // the sharded step's per-block histograms (kept between its two launches)
  off += sharded ? align256((size_t)P->grid * G * kHistStride * sizeof(uint32_t)) : 0;
  P->total = off;
  return ADAMAS_OK;
}

// Plans of the shapes seen so far, per device (a decode loop calls with the same
// shape every step: after the first call, planning is one table lookup).
struct PlanKey {
  int B, Hq, Hkv;
  int64_t Nmax;
  int mode;
};
constexpr int kPlanCache = 32;
struct PlanCache {
  PlanKey key[kPlanCache];
  Plan plan[kPlanCache];
  int n = 0, next = 0;
};
static PlanCache g_plans[kMaxDevices];

static int make_plan(int B, int Hq, int Hkv, int64_t Nmax, int mode, DeviceInfo& dev, int devno, Plan* P) {
  PlanCache& pc = g_plans[devno];
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int i = 0; i < pc.n; ++i) {
      const PlanKey& k = pc.key[i];
      if (k.B == B && k.Hq == Hq && k.Hkv == Hkv && k.Nmax == Nmax && k.mode == mode) {
        *P = pc.plan[i];
        return ADAMAS_OK;
      }
    }
  }
  const int rc = make_plan_uncached(B, Hq, Hkv, Nmax, mode, dev, P);
  if (rc != ADAMAS_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mutex);
  const int slot = pc.n < kPlanCache ? pc.n++ : (pc.next++ % kPlanCache);
  pc.key[slot] = PlanKey{B, Hq, Hkv, Nmax, mode};
  pc.plan[slot] = *P;
  return ADAMAS_OK;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int launch_decode(const DecodeParams& prm, const Plan& P, int mode, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // the launch may begin while the previous kernel of the stream finishes: the
  // kernel waits for it (griddepcontrol.wait) before touching global memory
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = decode_launch_for(P.G, &cfg, prm, P.smem_d, mode);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

// Argument checks of a decode call (before anything is enqueued).  Fills *Nmax_out
// with the tokens a sequence can hold (paged: max_pages * page_size).
static int check_decode_args(const adamas_decode_args& a, int64_t* Nmax_out) {
  const bool paged = a.block_table != nullptr;
  int64_t Nmax = a.Nmax;
  if (paged) {
    if (a.page_size < 1 || a.max_pages < 1 || a.n_pages < 1) return ADAMAS_ERR_INVALID_ARG;
    Nmax = (int64_t)a.max_pages * a.page_size;
    if (Nmax > INT32_MAX || a.n_pages * a.Hkv * (int64_t)a.page_size > INT32_MAX) return ADAMAS_ERR_UNSUPPORTED;
    if (!aligned(a.block_table, 4)) return ADAMAS_ERR_INVALID_ARG;
  }
  *Nmax_out = Nmax;
  int rc = check_shape(a.B, a.Hq, a.Hkv, Nmax, a.d, a.budget);
  if (rc != ADAMAS_OK) return rc;
  if (a.policy != ADAMAS_SELECT_PER_HEAD && a.policy != ADAMAS_SELECT_GROUP_SHARED) return ADAMAS_ERR_INVALID_ARG;
  if (a.policy == ADAMAS_SELECT_GROUP_SHARED && a.budget > kKeptCap) return ADAMAS_ERR_UNSUPPORTED;
  if (a.n_sink < 0 || a.n_recent < 0) return ADAMAS_ERR_INVALID_ARG;
  if (a.B == 0) return ADAMAS_OK;
  if (!a.q || !a.seq_lens || !a.out || (a.budget > 0 && !a.idx)) return ADAMAS_ERR_INVALID_ARG;
  if (Nmax > 0 && (!a.codes || !a.K || !a.V)) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(a.q, 16) || !aligned(a.codes, 32) || !aligned(a.K, 16) || !aligned(a.V, 16) || !aligned(a.out, 16) ||
      !aligned(a.idx, 4) || !aligned(a.seq_lens, 4))
    return ADAMAS_ERR_INVALID_ARG;
  if ((a.k_new == nullptr) != (a.v_new == nullptr)) return ADAMAS_ERR_INVALID_ARG;
  if (a.k_new && (!a.append_pos || !aligned(a.k_new, 16) || !aligned(a.v_new, 16))) return ADAMAS_ERR_INVALID_ARG;
  if (a.append_pos && !aligned(a.append_pos, 4)) return ADAMAS_ERR_INVALID_ARG;
  return ADAMAS_OK;
}

// Test hook of adamas_debug_withhold_stage: the stage whose copy the next steps
// never issue (-1: none).
static std::atomic<int> g_withhold{-1};

// The kernel instance a call needs: group-shared, general (any option), or plain.
static int decode_mode(const adamas_decode_args& a) {
  if (a.policy == ADAMAS_SELECT_GROUP_SHARED) return kModeShared;
  if (a.block_table || a.k_new || a.n_sink > 0 || a.n_recent > 0 || g_withhold.load() >= 0) return kModeGeneral;
  return kModePlain;
}

// Enqueue the decode kernel with its scratch at `ws` (laid out by `P`).
static int enqueue_decode(const adamas_decode_args& a, int64_t Nmax, unsigned char* ws, const Plan& P,
                          cudaStream_t st) {
  DecodeParams prm = {};
  prm.q = static_cast<const uint16_t*>(a.q);
  prm.codes = a.codes;
  prm.K = static_cast<const uint16_t*>(a.K);
  prm.V = static_cast<const uint16_t*>(a.V);
  prm.seq_lens = a.seq_lens;
  prm.out = a.out;
  prm.idx = a.idx;
  prm.err = reinterpret_cast<uint32_t*>(ws + P.ctrl) + 2;
  prm.dglobal = P.smem_d ? nullptr : reinterpret_cast<uint16_t*>(ws + P.dspill);
  prm.codes_w = a.append_pos ? a.codes : nullptr;
  prm.append_pos = a.append_pos;
  prm.k_new = static_cast<const uint16_t*>(a.k_new);
  prm.v_new = static_cast<const uint16_t*>(a.v_new);
  prm.K_w = a.k_new ? static_cast<uint16_t*>(a.K) : nullptr;
  prm.V_w = a.k_new ? static_cast<uint16_t*>(a.V) : nullptr;
  prm.table = a.block_table;
  prm.n_pages = a.block_table ? a.n_pages : 0;
  prm.page_size = a.block_table ? a.page_size : 1;
  prm.max_pages = a.block_table ? a.max_pages : 0;
  prm.n_sink = a.n_sink;
  prm.n_recent = a.n_recent;
  prm.withhold = g_withhold.load();
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.Nmax = Nmax;
  prm.budget = a.budget;
  prm.cluster = P.cluster;
  prm.nstages = P.nstages;
  prm.dstride = P.dstride;
  return launch_decode(prm, P, decode_mode(a), st);
}

// Few long heads (too few clusters for the SMs): the plain step splits every
// (b, kv head) into S slices inside the GPU -- the sharded step's two launches with
// vslices = S and a merge of the S softmax states (defined with the sequence-sharded
// step below).
struct SlicePlan {
  int S = 1;
  Plan P;
  size_t hist_off = 0, part_off = 0, total = 0;
};
static int slice_plan(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget, const Plan& P0, DeviceInfo& dev,
                      SlicePlan* out);
static int enqueue_sliced(const adamas_decode_args& a, int64_t Nmax, const SlicePlan& SP, cudaStream_t st);

// A decode call on a caller workspace: checks, plan, launch.
static int decode_with_workspace(const adamas_decode_args& a, cudaStream_t st) {
  int64_t Nmax = 0;
  int rc = check_decode_args(a, &Nmax);
  if (rc != ADAMAS_OK || a.B == 0) return rc;
  DeviceInfo* dev = nullptr;
  int devno = 0;
  if ((rc = device_info(&dev, &devno)) != ADAMAS_OK) return rc;
  Plan P;
  const int mode = decode_mode(a);
  if ((rc = make_plan(a.B, a.Hq, a.Hkv, Nmax, mode, *dev, devno, &P)) != ADAMAS_OK) return rc;
  if (mode == kModePlain) {
    SlicePlan SP;
    if ((rc = slice_plan(a.B, a.Hq, a.Hkv, Nmax, a.d, a.budget, P, *dev, &SP)) != ADAMAS_OK) return rc;
    if (SP.S > 1) {
      if (!a.workspace || a.workspace_bytes < SP.total || !aligned(a.workspace, 16)) return ADAMAS_ERR_WORKSPACE;
      return enqueue_sliced(a, Nmax, SP, st);
    }
  }
  if (!a.workspace || a.workspace_bytes < P.total || !aligned(a.workspace, 16)) return ADAMAS_ERR_WORKSPACE;
  return enqueue_decode(a, Nmax, static_cast<unsigned char*>(a.workspace), P, st);
}

template <int G>
static void launch_score(dim3 grid, cudaStream_t st, const uint16_t* q, const uint8_t* codes, const int32_t* lens,
                         int Hq, int Hkv, int64_t Nmax, uint16_t* dist) {
  score_kernel<G><<<grid, kScoreThreads, 0, st>>>(q, codes, lens, Hq, Hkv, Nmax, dist);
}

}  // namespace adamas

using namespace adamas;

extern "C" {

const char* adamas_status_string(int status) {
  switch (status) {
    case ADAMAS_OK: return "ok";
    case ADAMAS_ERR_INVALID_ARG: return "invalid argument";
    case ADAMAS_ERR_UNSUPPORTED: return "unsupported size or configuration";
    case ADAMAS_ERR_WORKSPACE: return "workspace missing or too small";
    case ADAMAS_ERR_CUDA: return "CUDA runtime error";
    case ADAMAS_ERR_DEVICE: return "device error word set";
    default: return "unknown status";
  }
}

int adamas_version(void) { return 200; }

const char* adamas_last_error_string(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

size_t adamas_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget) {
  if (check_shape(B, Hq, Hkv, Nmax, d, budget) != ADAMAS_OK) return 0;
  DeviceInfo* dev = nullptr;
  int devno = 0;
  if (device_info(&dev, &devno) != ADAMAS_OK) return 0;
  Plan P;
  if (make_plan(B, Hq, Hkv, Nmax, kModePlain, *dev, devno, &P) != ADAMAS_OK) return 0;
  SlicePlan SP;
  if (slice_plan(B, Hq, Hkv, Nmax, d, budget, P, *dev, &SP) != ADAMAS_OK) return 0;
  return SP.S > 1 && SP.total > P.total ? SP.total : P.total;
}

int adamas_workspace_init(void* workspace, size_t workspace_bytes, adamas_stream_t stream) {
  if (!workspace || workspace_bytes == 0) return ADAMAS_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

int adamas_encode_keys(const void* K, uint8_t* codes, const int32_t* pos_begin, int count, int B, int Hkv,
                       int64_t Nmax, int d, adamas_stream_t stream) {
  // no batch limit here: the pages of a paged cache are encoded as B = n_pages sequences
  if (B < 0 || Hkv <= 0 || Nmax < 0 || count < 0) return ADAMAS_ERR_INVALID_ARG;
  if (d != kDim) return ADAMAS_ERR_UNSUPPORTED;
  if (Nmax > INT32_MAX || (int64_t)B * Hkv > INT32_MAX) return ADAMAS_ERR_UNSUPPORTED;
  if (B == 0 || count == 0 || Nmax == 0) return ADAMAS_OK;
  if (!K || !codes || !aligned(K, 16) || !aligned(codes, 32)) return ADAMAS_ERR_INVALID_ARG;
  if (pos_begin && !aligned(pos_begin, 4)) return ADAMAS_ERR_INVALID_ARG;
  const int64_t nvec = (int64_t)count * B * Hkv;
  if (nvec <= kEncWarpMaxVectors) {
    const int per_block = kEncWarpThreads / 32;
    encode_keys_warp_kernel<<<(unsigned)((nvec + per_block - 1) / per_block), kEncWarpThreads, 0,
                              (cudaStream_t)stream>>>(static_cast<const uint16_t*>(K), codes, pos_begin, count, Hkv,
                                                      Nmax, nvec);
  } else {
    DeviceInfo* dev = nullptr;
    int rc2 = device_info(&dev);
    if (rc2 != ADAMAS_OK) return rc2;
    if ((rc2 = encoder_attrs(*dev)) != ADAMAS_OK) return rc2;
    const int tiles_per_head = (int)(((int64_t)count + 31) / 32);
    const int64_t ntiles = (int64_t)tiles_per_head * B * Hkv;
    if (ntiles > INT32_MAX) return ADAMAS_ERR_UNSUPPORTED;
    const int64_t want = (ntiles + kEncWarps - 1) / kEncWarps;
    const int64_t cap = (int64_t)dev->sms * dev->enc_blocks_per_sm;
    const unsigned grid = (unsigned)(want < cap ? want : cap);
    encode_keys_kernel<<<grid, kEncThreads, kEncSmem, (cudaStream_t)stream>>>(
        static_cast<const uint16_t*>(K), codes, pos_begin, count, Hkv, Nmax, tiles_per_head, B * Hkv);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

// The plain calls below are adamas_decode_step_ex with the optional fields unset.
static adamas_decode_args plain_args(const void* q, const uint8_t* codes, const void* K, const void* V,
                                     const int32_t* seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d, int budget,
                                     float* out, int32_t* idx, void* workspace, size_t workspace_bytes) {
  adamas_decode_args a;
  memset(&a, 0, sizeof a);
  a.q = q;
  a.codes = const_cast<uint8_t*>(codes);
  a.K = const_cast<void*>(K);
  a.V = const_cast<void*>(V);
  a.seq_lens = seq_lens;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nmax = Nmax;
  a.d = d;
  a.budget = budget;
  a.out = out;
  a.idx = idx;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.policy = ADAMAS_SELECT_PER_HEAD;
  return a;
}

int adamas_decode_step(const void* q, const uint8_t* codes, const void* K, const void* V, const int32_t* seq_lens,
                       int B, int Hq, int Hkv, int64_t Nmax, int d, int budget, float* out, int32_t* idx,
                       void* workspace, size_t workspace_bytes, adamas_stream_t stream) {
  const adamas_decode_args a =
      plain_args(q, codes, K, V, seq_lens, B, Hq, Hkv, Nmax, d, budget, out, idx, workspace, workspace_bytes);
  return decode_with_workspace(a, (cudaStream_t)stream);
}

int adamas_decode_step_append(const void* q, uint8_t* codes, const void* K, const void* V, const int32_t* seq_lens,
                              const int32_t* append_pos, int B, int Hq, int Hkv, int64_t Nmax, int d, int budget,
                              float* out, int32_t* idx, void* workspace, size_t workspace_bytes,
                              adamas_stream_t stream) {
  if (B > 0 && !append_pos) return ADAMAS_ERR_INVALID_ARG;
  adamas_decode_args a =
      plain_args(q, codes, K, V, seq_lens, B, Hq, Hkv, Nmax, d, budget, out, idx, workspace, workspace_bytes);
  a.append_pos = append_pos;
  return decode_with_workspace(a, (cudaStream_t)stream);
}

void adamas_debug_withhold_stage(int stage) { g_withhold.store(stage < 0 ? -1 : stage); }

int adamas_decode_step_ex(const adamas_decode_args* args, adamas_stream_t stream) {
  if (!args) return ADAMAS_ERR_INVALID_ARG;
  return decode_with_workspace(*args, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ sequence-sharded step
static_assert(kHistStride == ADAMAS_HIST_STRIDE && kPartial == ADAMAS_PARTIAL_FLOATS,
              "the exchange layouts of the header");
// Both halves use one plan (the score half's), so that block i of the attend half
// finds the distances and histograms that block i of the score half left.
static int shard_plan(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget, Plan* P) {
  int rc = check_shape(B, Hq, Hkv, Nmax, d, budget);
  if (rc != ADAMAS_OK) return rc;
  DeviceInfo* dev = nullptr;
  int devno = 0;
  if ((rc = device_info(&dev, &devno)) != ADAMAS_OK) return rc;
  if ((rc = make_plan(B, Hq, Hkv, Nmax, kModeShardScore, *dev, devno, P)) != ADAMAS_OK) return rc;
  // the attend half's instance: the same shared memory and cluster shape
  const void* fn = decode_fn_for(P->G, false, kModeShardAttend);
  if ((rc = kernel_attrs(*dev, fn, P->G, false, kModeShardAttend)) != ADAMAS_OK) return rc;
  int n = 0;
  if ((rc = active_clusters(*dev, fn, P->cluster, P->smem, &n)) != ADAMAS_OK) return rc;
  return n >= 1 ? ADAMAS_OK : ADAMAS_ERR_UNSUPPORTED;
}

static void shard_params(DecodeParams& prm, const Plan& P, unsigned char* ws, const void* q, const int32_t* seq_lens,
                         int B, int Hq, int Hkv, int64_t Nmax, int budget) {
  prm.q = static_cast<const uint16_t*>(q);
  prm.seq_lens = seq_lens;
  prm.err = reinterpret_cast<uint32_t*>(ws + P.ctrl) + 2;
  prm.dglobal = reinterpret_cast<uint16_t*>(ws + P.dspill);
  prm.blk_hist = reinterpret_cast<uint32_t*>(ws + P.bhist);
  prm.withhold = -1;
  prm.page_size = 1;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nmax = Nmax;
  prm.budget = budget;
  prm.cluster = P.cluster;
  prm.nstages = P.nstages;
  prm.dstride = P.dstride;
  prm.shard_world = 1;
}

size_t adamas_shard_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget) {
  Plan P;
  if (shard_plan(B, Hq, Hkv, Nmax, d, budget, &P) != ADAMAS_OK) return 0;
  return P.total;
}

int adamas_shard_score(const void* q, const uint8_t* codes, const int32_t* seq_lens, int B, int Hq, int Hkv,
                       int64_t Nmax, int d, int budget, uint32_t* hist, void* workspace, size_t workspace_bytes,
                       adamas_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, Nmax, d, budget);
  if (rc != ADAMAS_OK || B == 0) return rc;
  if (!q || !seq_lens || !hist || (Nmax > 0 && !codes)) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(codes, 32) || !aligned(seq_lens, 4) || !aligned(hist, 4))
    return ADAMAS_ERR_INVALID_ARG;
  Plan P;
  if ((rc = shard_plan(B, Hq, Hkv, Nmax, d, budget, &P)) != ADAMAS_OK) return rc;
  if (!workspace || workspace_bytes < P.total || !aligned(workspace, 16)) return ADAMAS_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)B * Hq * kHistStride * sizeof(uint32_t), st);
  if (e != cudaSuccess) return cuda_fail(e);
  DecodeParams prm = {};
  shard_params(prm, P, static_cast<unsigned char*>(workspace), q, seq_lens, B, Hq, Hkv, Nmax, budget);
  prm.codes = codes;
  prm.shard_hist = hist;
  return launch_decode(prm, P, kModeShardScore, st);
}

int adamas_shard_attend(const void* q, const void* K, const void* V, const int32_t* seq_lens, int B, int Hq, int Hkv,
                        int64_t Nmax, int d, int budget, const uint32_t* hist_all, int world, int rank,
                        float* partial, int32_t* idx, void* workspace, size_t workspace_bytes,
                        adamas_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, Nmax, d, budget);
  if (rc != ADAMAS_OK || B == 0) return rc;
  if (world < 1 || rank < 0 || rank >= world) return ADAMAS_ERR_INVALID_ARG;
  if (!q || !seq_lens || !hist_all || !partial || (budget > 0 && !idx) || (Nmax > 0 && (!K || !V)))
    return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(seq_lens, 4) || !aligned(hist_all, 4) ||
      !aligned(partial, 16) || !aligned(idx, 4))
    return ADAMAS_ERR_INVALID_ARG;
  Plan P;
  if ((rc = shard_plan(B, Hq, Hkv, Nmax, d, budget, &P)) != ADAMAS_OK) return rc;
  if (!workspace || workspace_bytes < P.total || !aligned(workspace, 16)) return ADAMAS_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  if (budget > 0) {  // slots of other slices' tokens and past k_eff stay -1
    const cudaError_t e = cudaMemsetAsync(idx, 0xFF, (size_t)B * Hq * budget * sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  DecodeParams prm = {};
  shard_params(prm, P, static_cast<unsigned char*>(workspace), q, seq_lens, B, Hq, Hkv, Nmax, budget);
  prm.K = static_cast<const uint16_t*>(K);
  prm.V = static_cast<const uint16_t*>(V);
  prm.idx = idx;
  prm.hist_all = hist_all;
  prm.partial = partial;
  prm.shard_rank = rank;
  prm.shard_world = world;
  return launch_decode(prm, P, kModeShardAttend, st);
}

int adamas_merge_partials(const float* partials, int n, int B, int Hq, float* out, adamas_stream_t stream) {
  if (n < 1 || B < 0 || Hq < 0) return ADAMAS_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)B * Hq;
  if (rows == 0) return ADAMAS_OK;
  if (rows > INT32_MAX) return ADAMAS_ERR_UNSUPPORTED;
  if (!partials || !out || !aligned(partials, 16) || !aligned(out, 16)) return ADAMAS_ERR_INVALID_ARG;
  merge_partials_kernel<<<(unsigned)rows, kDim, 0, (cudaStream_t)stream>>>(partials, n, rows, out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

}  // extern "C"

namespace adamas {

constexpr int64_t kSliceMinTokens = 65536;  // shorter contexts stay one launch (fixed costs dominate)
constexpr int kMaxSlices = 8;

static int slice_plan(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget, const Plan& P0, DeviceInfo& dev,
                      SlicePlan* out) {
  out->S = 1;
  if (Nmax < kSliceMinTokens || (int64_t)P0.grid * 4 >= (int64_t)dev.sms * 3) return ADAMAS_OK;
  int best = P0.grid;
  for (int S = 2; S <= kMaxSlices; ++S) {
    if ((int64_t)B * Hkv * S > 65535) break;
    Plan P;
    // S virtual heads of ceil(Nmax / S) tokens per (b, kv head); the query heads follow
    if (shard_plan(B, Hq * S, Hkv * S, (Nmax + S - 1) / S, d, budget, &P) != ADAMAS_OK) continue;
    if (P.grid > best + best / 8) {  // two more launches are worth it only for clearly more blocks
      best = P.grid;
      out->S = S;
      out->P = P;
    }
  }
  if (out->S > 1) {
    const size_t rows = (size_t)B * Hq * out->S;
    out->hist_off = align256(out->P.total);
    out->part_off = out->hist_off + align256(rows * kHistStride * sizeof(uint32_t));
    out->total = out->part_off + align256(rows * kPartial * sizeof(float));
  }
  return ADAMAS_OK;
}

static int enqueue_sliced(const adamas_decode_args& a, int64_t Nmax, const SlicePlan& SP, cudaStream_t st) {
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + SP.hist_off);
  float* part = reinterpret_cast<float*>(ws + SP.part_off);
  const size_t rows = (size_t)a.B * a.Hq;
  cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)SP.S * rows * kHistStride * sizeof(uint32_t), st);
  if (e == cudaSuccess && a.budget > 0) e = cudaMemsetAsync(a.idx, 0xFF, rows * a.budget * sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e);
  DecodeParams prm = {};
  shard_params(prm, SP.P, ws, a.q, a.seq_lens, a.B, a.Hq, a.Hkv, Nmax, a.budget);
  prm.vslices = SP.S;
  prm.codes = a.codes;
  prm.K = static_cast<const uint16_t*>(a.K);  // the appended key is encoded from its K row
  prm.V = static_cast<const uint16_t*>(a.V);
  prm.shard_hist = hist;
  prm.append_pos = a.append_pos;
  prm.codes_w = a.append_pos ? a.codes : nullptr;
  int rc = launch_decode(prm, SP.P, kModeShardScore, st);
  if (rc != ADAMAS_OK) return rc;
  DecodeParams prm2 = {};
  shard_params(prm2, SP.P, ws, a.q, a.seq_lens, a.B, a.Hq, a.Hkv, Nmax, a.budget);
  prm2.vslices = SP.S;
  prm2.K = static_cast<const uint16_t*>(a.K);
  prm2.V = static_cast<const uint16_t*>(a.V);
  prm2.idx = a.idx;
  prm2.hist_all = hist;
  prm2.partial = part;
  if ((rc = launch_decode(prm2, SP.P, kModeShardAttend, st)) != ADAMAS_OK) return rc;
  merge_partials_kernel<<<(unsigned)rows, kDim, 0, st>>>(part, SP.S, (int64_t)rows, a.out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

}  // namespace adamas

extern "C" {

int adamas_score(const void* q, const uint8_t* codes, const int32_t* seq_lens, int B, int Hq, int Hkv, int64_t Nmax,
                 int d, uint16_t* dist, adamas_stream_t stream) {
  const int rc = check_shape(B, Hq, Hkv, Nmax, d, 0);
  if (rc != ADAMAS_OK) return rc;
  if (B == 0 || Nmax == 0) return ADAMAS_OK;
  if (!q || !codes || !seq_lens || !dist) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(codes, 32) || !aligned(seq_lens, 4) || !aligned(dist, 2))
    return ADAMAS_ERR_INVALID_ARG;
  const int64_t per_block = (int64_t)kScoreThreads * kScoreUnroll;
  const dim3 grid((unsigned)((Nmax + per_block - 1) / per_block), (unsigned)(B * Hkv));
  cudaStream_t st = (cudaStream_t)stream;
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  switch (Hq / Hkv) {
    case 1: launch_score<1>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 2: launch_score<2>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 3: launch_score<3>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 4: launch_score<4>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 5: launch_score<5>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 6: launch_score<6>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 7: launch_score<7>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    case 8: launch_score<8>(grid, st, qq, codes, seq_lens, Hq, Hkv, Nmax, dist); break;
    default: return ADAMAS_ERR_UNSUPPORTED;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

int adamas_get_device_error(const void* workspace, size_t workspace_bytes, uint32_t* error_word,
                            adamas_stream_t stream) {
  if (!workspace || !error_word || workspace_bytes < 64 * sizeof(uint32_t)) return ADAMAS_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&word, static_cast<const uint32_t*>(workspace) + 2, sizeof word,
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  *error_word = word;
  return word == 0 ? ADAMAS_OK : ADAMAS_ERR_DEVICE;
}

}  // extern "C"

// ------------------------------------------------------------------ decode step without a caller workspace
// Some callers cannot allocate device memory at the point where they decode: a
// custom allocator that must not be re-entered from inside a serving loop, a
// framework hook that runs with allocation forbidden, or a host program that only
// ever receives pointers to memory someone else owns.  adamas_decode_step_static
// serves them: it uses a fixed scratch array that the library itself holds in
// every device's global memory (a file-scope __device__ array, reserved when the
// library's module is loaded onto a device and kept until the process exits),
// so it needs no workspace argument and calls no allocator.
namespace adamas {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB on every device that loads the library

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

static std::mutex g_static_mutex;

// Driver calls reached through the runtime's entry-point query (the library links
// only the runtime): the current context and its process-unique id.
typedef int (*CtxGetCurrentFn)(void** ctx);
typedef int (*CtxGetIdFn)(void* ctx, unsigned long long* id);

static int driver_fn(const char* name, void** fn) {
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  const cudaError_t e = cudaGetDriverEntryPointByVersion(name, fn, 12000, cudaEnableDefault, &q);
  if (e != cudaSuccess) return cuda_fail(e);
  return q == cudaDriverEntryPointSuccess && *fn ? ADAMAS_OK : ADAMAS_ERR_UNSUPPORTED;
}

// Device address of g_static_scratch in the current context.  In host code the
// array's name is only a host-side stand-in: the address is looked up with the
// context current and cached under the context's id, which the driver never
// reuses within a process.  A context created later (after cudaDeviceReset, or
// another context made current) has another id and gets its own lookup, so a
// cached address never outlives the context it was taken in.
static int static_scratch(void** out) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  constexpr int kSlots = 16;
  static unsigned long long ids[kSlots] = {};
  static void* ptrs[kSlots] = {};
  static int next = 0;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  int rc;
  if (!get_current && (rc = driver_fn("cuCtxGetCurrent", reinterpret_cast<void**>(&get_current))) != ADAMAS_OK)
    return rc;
  if (!get_id && (rc = driver_fn("cuCtxGetId", reinterpret_cast<void**>(&get_id))) != ADAMAS_OK) return rc;
  void* ctx = nullptr;
  if (get_current(&ctx) != 0 || ctx == nullptr) {  // none yet: the runtime makes the device's primary context current
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (get_current(&ctx) != 0 || ctx == nullptr) return ADAMAS_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != 0) return ADAMAS_ERR_CUDA;
  for (int i = 0; i < kSlots; ++i)
    if (ptrs[i] && ids[i] == id) {
      *out = ptrs[i];
      return ADAMAS_OK;
    }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  ids[next] = id;
  ptrs[next] = p;
  next = (next + 1) % kSlots;
  *out = p;
  return ADAMAS_OK;
}

}  // namespace adamas

extern "C" int adamas_decode_step_static(const void* q, const uint8_t* codes, const void* K, const void* V,
                                         const int32_t* seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d,
                                         int budget, float* out, int32_t* idx, adamas_stream_t stream) {
  const adamas_decode_args a = plain_args(q, codes, K, V, seq_lens, B, Hq, Hkv, Nmax, d, budget, out, idx, nullptr, 0);
  int64_t Nm = 0;
  int rc = check_decode_args(a, &Nm);
  if (rc != ADAMAS_OK || B == 0) return rc;
  DeviceInfo* dev = nullptr;
  int devno = 0;
  if ((rc = device_info(&dev, &devno)) != ADAMAS_OK) return rc;
  Plan P;
  if ((rc = make_plan(B, Hq, Hkv, Nm, kModePlain, *dev, devno, &P)) != ADAMAS_OK) return rc;
  if (P.total > kStaticScratchBytes) return ADAMAS_ERR_WORKSPACE;  // sizes beyond the fixed scratch
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch)) != ADAMAS_OK) return rc;
  // The scratch keeps whatever the previous call left; the error word must start
  // at zero.
  cudaStream_t st = (cudaStream_t)stream;
  const cudaError_t e = cudaMemsetAsync(scratch, 0, P.dspill, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return enqueue_decode(a, Nm, static_cast<unsigned char*>(scratch), P, st);
}

extern "C" int adamas_static_device_error(uint32_t* error_word, adamas_stream_t stream) {
  if (!error_word) return ADAMAS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = adamas::static_scratch(&scratch);
  if (rc != ADAMAS_OK) return rc;
  return adamas_get_device_error(scratch, adamas::kStaticScratchBytes, error_word, stream);
}
