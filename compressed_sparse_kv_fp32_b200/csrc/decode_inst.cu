// Instances of the decode kernel for one group size (ADAMAS_DECODE_G, set by the
// build), each kernel mode and distance placement, and their launch.  One
// translation unit per group size so that the instances compile in parallel.
#include "decode_ext.cuh"
#include "decode_plain.cuh"

#ifndef ADAMAS_DECODE_G
#error "ADAMAS_DECODE_G must be defined"
#endif

namespace adamas {

#define ADAMAS_CAT2(a, b) a##b
#define ADAMAS_CAT(a, b) ADAMAS_CAT2(a, b)

template <int MODE>
static const void* fn_of(bool smem_d) {
  constexpr int G = ADAMAS_DECODE_G;
  return smem_d ? reinterpret_cast<const void*>(&decode_step_ext_kernel<G, true, MODE>)
                : reinterpret_cast<const void*>(&decode_step_ext_kernel<G, false, MODE>);
}

template <int MODE>
static cudaError_t launch_of(const cudaLaunchConfig_t* cfg, const DecodeParams& prm, bool smem_d) {
  constexpr int G = ADAMAS_DECODE_G;
  return smem_d ? cudaLaunchKernelEx(cfg, decode_step_ext_kernel<G, true, MODE>, prm)
                : cudaLaunchKernelEx(cfg, decode_step_ext_kernel<G, false, MODE>, prm);
}

const void* ADAMAS_CAT(decode_fn_g, ADAMAS_DECODE_G)(bool smem_d, int mode) {
  constexpr int G = ADAMAS_DECODE_G;
  switch (mode) {
    case kModePlain:
      return smem_d ? reinterpret_cast<const void*>(&decode_step_kernel<G, true>)
                    : reinterpret_cast<const void*>(&decode_step_kernel<G, false>);
    case kModeGeneral: return fn_of<kModeGeneral>(smem_d);
    case kModeShared: return fn_of<kModeShared>(smem_d);
    // the sharded step keeps its distances in the workspace
    case kModeShardScore: return reinterpret_cast<const void*>(&decode_step_ext_kernel<G, false, kModeShardScore>);
    default: return reinterpret_cast<const void*>(&decode_step_ext_kernel<G, false, kModeShardAttend>);
  }
}

cudaError_t ADAMAS_CAT(decode_launch_g, ADAMAS_DECODE_G)(const cudaLaunchConfig_t* cfg, const DecodeParams& prm,
                                                         bool smem_d, int mode) {
  constexpr int G = ADAMAS_DECODE_G;
  switch (mode) {
    case kModePlain:
      return smem_d ? cudaLaunchKernelEx(cfg, decode_step_kernel<G, true>, prm)
                    : cudaLaunchKernelEx(cfg, decode_step_kernel<G, false>, prm);
    case kModeGeneral: return launch_of<kModeGeneral>(cfg, prm, smem_d);
    case kModeShared: return launch_of<kModeShared>(cfg, prm, smem_d);
    case kModeShardScore: return cudaLaunchKernelEx(cfg, decode_step_ext_kernel<G, false, kModeShardScore>, prm);
    default: return cudaLaunchKernelEx(cfg, decode_step_ext_kernel<G, false, kModeShardAttend>, prm);
  }
}

}  // namespace adamas
