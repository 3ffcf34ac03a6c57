// C ABI of the ADAMAS sparse decode library (declared in include/adamas.h):
// argument checks, workspace layout, and the launches of the sm_100a kernels.
//
// Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
// §2.1 Hadamard rotation, §2.2 dynamic 2-bit bucketing, §3.1 packed code cache,
// §2.3 Manhattan-distance scoring, §5.2 token budget.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/adamas.h"
#include "common.cuh"
#include "decode.cuh"
#include "encode.cuh"
#include "score.cuh"

namespace adamas {

// ------------------------------------------------------------------ key encoder
constexpr int kEncThreads = 128;       // one vector per thread, one tile of 128 positions per block
constexpr int kEncRowWords = 68;       // 64 words of bf16 + 4 words of padding (bank spread)

__global__ void __launch_bounds__(kEncThreads) encode_keys_kernel(const uint16_t* __restrict__ K,
                                                                  uint8_t* __restrict__ codes,
                                                                  const int32_t* __restrict__ pos_begin,
                                                                  int count, int Hkv, int64_t Nmax) {
  __shared__ __align__(16) uint32_t tile[kEncThreads * kEncRowWords];
  const int tid = threadIdx.x;
  const int hk = blockIdx.y;
  const int b = hk / Hkv;
  const int64_t p0 = pos_begin ? (int64_t)pos_begin[b] : 0;
  const int64_t first = (int64_t)blockIdx.x * kEncThreads;
  const uint16_t* kbase = K + (int64_t)hk * Nmax * kDim;

  // coalesced 16-byte loads of the tile's rows into padded shared memory
#pragma unroll 4
  for (int i = tid; i < kEncThreads * 16; i += kEncThreads) {
    const int row = i >> 4, ch = i & 15;
    const int64_t r = first + row, pos = p0 + r;
    if (r < count && pos >= 0 && pos < Nmax) {
      const uint4 v = *reinterpret_cast<const uint4*>(kbase + pos * kDim + ch * 8);
      *reinterpret_cast<uint4*>(&tile[row * kEncRowWords + ch * 4]) = v;
    }
  }
  __syncthreads();

  const int64_t r = first + tid, pos = p0 + r;
  if (r >= count || pos < 0 || pos >= Nmax) return;
  float v[kDim];
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) {
    const uint4 w = *reinterpret_cast<const uint4*>(&tile[tid * kEncRowWords + ch * 4]);
    v[8 * ch + 0] = bf16_lo(w.x); v[8 * ch + 1] = bf16_hi(w.x);
    v[8 * ch + 2] = bf16_lo(w.y); v[8 * ch + 3] = bf16_hi(w.y);
    v[8 * ch + 4] = bf16_lo(w.z); v[8 * ch + 5] = bf16_hi(w.z);
    v[8 * ch + 6] = bf16_lo(w.w); v[8 * ch + 7] = bf16_hi(w.w);
  }
  fwht128_thread(v);
  uint32_t w[kCodeWords];
  bucket_pack_thread(v, w);
  uint4* dst = reinterpret_cast<uint4*>(codes + ((int64_t)hk * Nmax + pos) * kCodeBytes);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
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
  uint32_t qw[G][kCodeWords];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int w = 0; w < kCodeWords; ++w) qw[g][w] = sq[g * kCodeWords + w];
  const int64_t first = (int64_t)blockIdx.x * kScoreThreads * kScoreUnroll;
#pragma unroll
  for (int j = 0; j < kScoreUnroll; ++j) {
    const int64_t t = first + (int64_t)j * kScoreThreads + tid;
    if (t >= Nmax) break;
    uint32_t kc[kCodeWords], e[kCodeWords];
    if (t < len) {
      ld_stream_v8(codes + ((int64_t)hk * Nmax + t) * kCodeBytes, kc);
      key_odd_mask(kc, e);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint16_t d = t < len ? (uint16_t)l1_distance(kc, e, qw[g]) : (uint16_t)0xFFFF;
      dist[((int64_t)b * Hq + kvh * G + g) * Nmax + t] = d;
    }
  }
}

// ------------------------------------------------------------------ host side
struct DeviceInfo {
  int sms = 0;
  size_t smem_optin = 0;
  bool attrs_set[2][kMaxGroup + 1] = {};
};

static std::mutex g_mutex;
static DeviceInfo g_devices[64];
static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Record a failed CUDA call for adamas_last_error_string and map it to a status.
static int cuda_fail(cudaError_t e) {
  g_last_cuda_error = e;
  return ADAMAS_ERR_CUDA;
}

// Shared memory a block can use beyond the kernels' static shared memory.
constexpr size_t kStaticSmemReserve = 6144;  // static shared memory of the kernels + per-block system use

static int device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return ADAMAS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (d.sms == 0) {
    int sms = 0, optin = 0, per_sm = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess)
      return cuda_fail(e);
    // dynamic shared memory of one decode block when kBlocksPerSM share an SM
    size_t budget = (size_t)per_sm / kBlocksPerSM;
    if (budget > (size_t)optin) budget = (size_t)optin;
    d.smem_optin = budget > kStaticSmemReserve ? budget - kStaticSmemReserve : 0;
    d.sms = sms;
  }
  *out = &d;
  return ADAMAS_OK;
}

struct WsLayout {
  size_t ctrl, head_done, hist, partial, dspill, total;
  int S;
  int64_t range_cap;
  bool smem_d;
  bool stage_in_d;
  int row_cap;
  size_t smem;
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

static int ws_layout(int B, int Hq, int Hkv, int64_t Nmax, int budget, const DeviceInfo& dev, WsLayout* L) {
  const int G = Hq / Hkv;
  const int64_t umax = (int64_t)B * Hkv * Nmax;
  int64_t want = (umax + 2047) / 2048;
  const int max_blocks = dev.sms * kBlocksPerSM < kMaxBlocks ? dev.sms * kBlocksPerSM : kMaxBlocks;
  L->S = (int)(want < 1 ? 1 : (want > max_blocks ? max_blocks : want));
  L->range_cap = umax > 0 ? (umax + L->S - 1) / L->S : 1;
  // With equal lengths the kernel may split over a multiple of the kv-head count
  // (each block within one head): its shares are at most ceil(Nmax / (S / heads)).
  const int64_t heads = (int64_t)B * Hkv;
  if (heads > 0 && heads <= L->S) {
    const int64_t per_head = L->S / heads;
    const int64_t r2 = (Nmax + per_head - 1) / per_head;
    if (r2 > L->range_cap) L->range_cap = r2;
  }
  if (L->range_cap >= (int64_t(1) << 23)) return ADAMAS_ERR_UNSUPPORTED;  // token offsets are packed in 23 bits
  // Distances in shared memory when they fit beside the smallest gather staging;
  // the staging then takes what is left (an even number of rows).
  const size_t fixed = DecodeSmem::fixed(B, G);
  const size_t dist = DecodeSmem::align128(DecodeSmem::dist(G, L->range_cap, true));
  L->smem_d = fixed + dist + (size_t)kMinRowsStaged * kRowBytes <= dev.smem_optin;
  const size_t left = dev.smem_optin - fixed - (L->smem_d ? dist : 0);
  if (dev.smem_optin < fixed + (size_t)kMinRowsStaged * kRowBytes) return ADAMAS_ERR_UNSUPPORTED;
  // Staging the gathered rows over the distance row keeps most of the SM's
  // unified L1/shared storage as L1 for the code stream.
  L->stage_in_d = L->smem_d && budget <= kMaxKept && DecodeSmem::dstride(L->range_cap) * 2 / kRowBytes >= 64;
  size_t rows = L->stage_in_d ? kMinRowsStaged : left / kRowBytes;  // small fallback area for short segments
  if (rows > (size_t)kMaxRowsStaged) rows = kMaxRowsStaged;
  L->row_cap = (int)(rows & ~(size_t)1);
  L->smem = DecodeSmem::total(B, G, L->range_cap, L->smem_d, L->row_cap);
  if (L->smem > dev.smem_optin) return ADAMAS_ERR_UNSUPPORTED;
  size_t off = 0;
  L->ctrl = off;      off += align256(64 * sizeof(uint32_t));
  L->head_done = off; off += align256((size_t)B * Hq * sizeof(uint32_t));
  L->hist = off;      off += align256((size_t)(L->S + B * Hkv) * G * kHistStride * sizeof(uint32_t));
  L->partial = off;   off += align256((size_t)(L->S + B * Hkv) * G * kPartial * sizeof(float));
  L->dspill = off;
  off += L->smem_d ? 0 : align256((size_t)L->S * G * DecodeSmem::dstride(L->range_cap) * sizeof(uint16_t));
  L->total = off;
  return ADAMAS_OK;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

template <int G>
static int launch_decode(const DecodeParams& prm, const WsLayout& L, DeviceInfo& dev, cudaStream_t stream) {
  auto kernel = prm.smem_d ? decode_step_kernel<G, true> : decode_step_kernel<G, false>;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev.attrs_set[prm.smem_d ? 1 : 0][G]) {
      const cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dev.smem_optin);
      if (e != cudaSuccess) return cuda_fail(e);
      dev.attrs_set[prm.smem_d ? 1 : 0][G] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)L.S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, prm);
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
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

int adamas_version(void) { return 100; }

const char* adamas_last_error_string(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

size_t adamas_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget) {
  if (check_shape(B, Hq, Hkv, Nmax, d, budget) != ADAMAS_OK) return 0;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != ADAMAS_OK) return 0;
  WsLayout L;
  if (ws_layout(B, Hq, Hkv, Nmax, budget, *dev, &L) != ADAMAS_OK) return 0;
  return L.total;
}

int adamas_workspace_init(void* workspace, size_t workspace_bytes, adamas_stream_t stream) {
  if (!workspace || workspace_bytes == 0) return ADAMAS_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

int adamas_encode_keys(const void* K, uint8_t* codes, const int32_t* pos_begin, int count, int B, int Hkv,
                       int64_t Nmax, int d, adamas_stream_t stream) {
  const int rc = check_shape(B, Hkv, Hkv, Nmax, d, 0);
  if (rc != ADAMAS_OK) return rc;
  if (count < 0) return ADAMAS_ERR_INVALID_ARG;
  if (B == 0 || count == 0 || Nmax == 0) return ADAMAS_OK;
  if (!K || !codes || !aligned(K, 16) || !aligned(codes, 32)) return ADAMAS_ERR_INVALID_ARG;
  if (pos_begin && !aligned(pos_begin, 4)) return ADAMAS_ERR_INVALID_ARG;
  const dim3 grid((unsigned)((count + kEncThreads - 1) / kEncThreads), (unsigned)(B * Hkv));
  const int64_t nvec = (int64_t)count * B * Hkv;
  if (nvec <= kEncWarpMaxVectors) {
    const int per_block = kEncWarpThreads / 32;
    encode_keys_warp_kernel<<<(unsigned)((nvec + per_block - 1) / per_block), kEncWarpThreads, 0,
                              (cudaStream_t)stream>>>(static_cast<const uint16_t*>(K), codes, pos_begin, count, Hkv,
                                                      Nmax, nvec);
  } else {
    encode_keys_kernel<<<grid, kEncThreads, 0, (cudaStream_t)stream>>>(
        static_cast<const uint16_t*>(K), codes, pos_begin, count, Hkv, Nmax);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return ADAMAS_OK;
}

int adamas_decode_step(const void* q, const uint8_t* codes, const void* K, const void* V, const int32_t* seq_lens,
                       int B, int Hq, int Hkv, int64_t Nmax, int d, int budget, float* out, int32_t* idx,
                       void* workspace, size_t workspace_bytes, adamas_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, Nmax, d, budget);
  if (rc != ADAMAS_OK) return rc;
  if (B == 0) return ADAMAS_OK;
  if (!q || !seq_lens || !out || (budget > 0 && !idx)) return ADAMAS_ERR_INVALID_ARG;
  if (Nmax > 0 && (!codes || !K || !V)) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(codes, 32) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) ||
      !aligned(idx, 4) || !aligned(seq_lens, 4))
    return ADAMAS_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != ADAMAS_OK) return rc;
  WsLayout L;
  if ((rc = ws_layout(B, Hq, Hkv, Nmax, budget, *dev, &L)) != ADAMAS_OK) return rc;
  if (!workspace || workspace_bytes < L.total || !aligned(workspace, 16)) return ADAMAS_ERR_WORKSPACE;

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  DecodeParams prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.codes = codes;
  prm.K = static_cast<const uint16_t*>(K);
  prm.V = static_cast<const uint16_t*>(V);
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.idx = idx;
  prm.ctrl = reinterpret_cast<uint32_t*>(ws + L.ctrl);
  prm.head_done = reinterpret_cast<uint32_t*>(ws + L.head_done);
  prm.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  prm.partial = reinterpret_cast<float*>(ws + L.partial);
  prm.dglobal = L.smem_d ? nullptr : reinterpret_cast<uint16_t*>(ws + L.dspill);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nmax = Nmax;
  prm.budget = budget;
  prm.S = L.S;
  prm.range_cap = L.range_cap;
  prm.smem_d = L.smem_d ? 1 : 0;
  prm.row_cap = L.row_cap;
  prm.stage_in_d = L.stage_in_d ? 1 : 0;

  cudaStream_t st = (cudaStream_t)stream;
  switch (Hq / Hkv) {
    case 1: rc = launch_decode<1>(prm, L, *dev, st); break;
    case 2: rc = launch_decode<2>(prm, L, *dev, st); break;
    case 3: rc = launch_decode<3>(prm, L, *dev, st); break;
    case 4: rc = launch_decode<4>(prm, L, *dev, st); break;
    case 5: rc = launch_decode<5>(prm, L, *dev, st); break;
    case 6: rc = launch_decode<6>(prm, L, *dev, st); break;
    case 7: rc = launch_decode<7>(prm, L, *dev, st); break;
    case 8: rc = launch_decode<8>(prm, L, *dev, st); break;
    default: rc = ADAMAS_ERR_UNSUPPORTED;
  }
  if (rc == ADAMAS_OK) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) rc = cuda_fail(e);
  }
  return rc;
}

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
static void* g_static_scratch_ptr[64] = {};

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
static int static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return ADAMAS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return ADAMAS_OK;
}

}  // namespace adamas

extern "C" int adamas_decode_step_static(const void* q, const uint8_t* codes, const void* K, const void* V,
                                         const int32_t* seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d,
                                         int budget, float* out, int32_t* idx, adamas_stream_t stream) {
  int rc = check_shape(B, Hq, Hkv, Nmax, d, budget);
  if (rc != ADAMAS_OK) return rc;
  if (B == 0) return ADAMAS_OK;
  if (!q || !seq_lens || !out || (budget > 0 && !idx)) return ADAMAS_ERR_INVALID_ARG;
  if (Nmax > 0 && (!codes || !K || !V)) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(codes, 32) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) ||
      !aligned(idx, 4) || !aligned(seq_lens, 4))
    return ADAMAS_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != ADAMAS_OK) return rc;
  WsLayout L;
  if ((rc = ws_layout(B, Hq, Hkv, Nmax, budget, *dev, &L)) != ADAMAS_OK) return rc;
  if (L.total > kStaticScratchBytes) return ADAMAS_ERR_WORKSPACE;  // sizes beyond the fixed scratch
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch)) != ADAMAS_OK) return rc;

  // The scratch keeps whatever the previous call left; the grid-wait counters,
  // the error word and the per-head tickets must start at zero.
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(scratch, 0, L.hist, st);
  if (e != cudaSuccess) return cuda_fail(e);

  unsigned char* ws = static_cast<unsigned char*>(scratch);
  DecodeParams prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.codes = codes;
  prm.K = static_cast<const uint16_t*>(K);
  prm.V = static_cast<const uint16_t*>(V);
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.idx = idx;
  prm.ctrl = reinterpret_cast<uint32_t*>(ws + L.ctrl);
  prm.head_done = reinterpret_cast<uint32_t*>(ws + L.head_done);
  prm.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  prm.partial = reinterpret_cast<float*>(ws + L.partial);
  prm.dglobal = L.smem_d ? nullptr : reinterpret_cast<uint16_t*>(ws + L.dspill);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nmax = Nmax;
  prm.budget = budget;
  prm.S = L.S;
  prm.range_cap = L.range_cap;
  prm.smem_d = L.smem_d ? 1 : 0;
  prm.row_cap = L.row_cap;
  prm.stage_in_d = L.stage_in_d ? 1 : 0;
  switch (Hq / Hkv) {
    case 1: rc = launch_decode<1>(prm, L, *dev, st); break;
    case 2: rc = launch_decode<2>(prm, L, *dev, st); break;
    case 3: rc = launch_decode<3>(prm, L, *dev, st); break;
    case 4: rc = launch_decode<4>(prm, L, *dev, st); break;
    case 5: rc = launch_decode<5>(prm, L, *dev, st); break;
    case 6: rc = launch_decode<6>(prm, L, *dev, st); break;
    case 7: rc = launch_decode<7>(prm, L, *dev, st); break;
    case 8: rc = launch_decode<8>(prm, L, *dev, st); break;
    default: rc = ADAMAS_ERR_UNSUPPORTED;
  }
  if (rc == ADAMAS_OK) {
    e = cudaGetLastError();
    if (e != cudaSuccess) rc = cuda_fail(e);
  }
  return rc;
}
