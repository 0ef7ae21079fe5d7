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

// The kept (BF16) blocks of every row, for attention over the NVFP4 keys.
struct KeptParams {
  const float* block_err;     // [rows][nb_stride]
  const int32_t* seq_lens;
  int32_t* kept;              // [rows][2], -1: none
  int rows, Hkv, nb_stride, n_keep;
};
cudaError_t launch_kept_blocks(const KeptParams& p, cudaStream_t s, bool pdl);

}  // namespace qs
