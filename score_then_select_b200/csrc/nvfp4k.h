// nvfp4k.h - the gather of the NVFP4 storage variant's attended keys (nvfp4k.cu).
#pragma once

#include "qs_internal.h"

namespace qs {

struct GatherNvParams {
  GatherParams base;          // selection, cache, compact buffers (as gather-then-attend)
  const uint8_t* codes;       // NVFP4 code pages
  const uint8_t* scales;      // UE4M3 scale pages
  const float* key_center;    // [batch][Hkv][d]
  const float* key_gscale;    // 1 float
  const float* block_err;     // [batch][Hkv][nb_stride], or nullptr
  int nb_stride, n_keep;
};

cudaError_t launch_gather_kv_nvfp4k(const Plan& pl, const GatherNvParams& p, cudaStream_t s);

}  // namespace qs
