// score_nvfp4.cu - NVFP4 centred-key scan (block-scaled FP4 tensor cores).
#include "qs_device.cuh"

namespace qs {

cudaError_t launch_score_nvfp4(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl) {
  return cudaErrorNotSupported;
}

}  // namespace qs
