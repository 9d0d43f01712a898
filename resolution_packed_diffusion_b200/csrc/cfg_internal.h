// cfg_internal.h -- the packed-CFG combine's launch interface, shared by the
// library's translation units. Not part of the public ABI (that is include/mf.h).
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf.h"

namespace mf {

// Row map of a packed-CFG combine: pair p writes output rows [out0[p],
// out0[p + 1]) from rows cond0[p] + i and uncond0[p] + i of v.
constexpr int kMaxCfgPairs = MF_MAX_SAMPLES / 2;
struct CfgTable {
  int32_t P;
  int32_t out0[kMaxCfgPairs + 1];
  int32_t cond0[kMaxCfgPairs];
  int32_t uncond0[kMaxCfgPairs];
};
cudaError_t launch_cfg_combine(const mf_bf16* v, const CfgTable& tab, int32_t C, float w,
                               mf_bf16* out, cudaStream_t st);

}  // namespace mf
