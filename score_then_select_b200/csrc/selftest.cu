// selftest.cu - diagnostic: a bounded wait that nothing can satisfy must give up and report.
//
// Every wait inside the library's kernels (mbarrier phases of the copy pipelines, the
// consumer groups' barriers) is bounded: after a fixed number of polls it records
// QS_ERR_DEVICE_TIMEOUT in the workspace status word and the kernel ends, so a lost arrival
// can never hang the GPU. This kernel runs the same bounded wait on an mbarrier phase that
// no thread ever completes, with a short limit, so a caller (and the tests) can check on a
// given GPU that the wait ends and that the context stays usable afterwards.
#include "qs_device.cuh"

namespace qs {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t* hdr, uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);            // one arrival expected; none ever comes
    fence_mbar_init();
  }
  __syncwarp();
  const bool done = mbar_wait(&bar, 0, polls);
  if (!done && threadIdx.x == 0) flag_error(hdr, QS_ERR_DEVICE_TIMEOUT, KID_SELFTEST, polls);
}

}  // namespace qs

using namespace qs;

extern "C" qs_status qs_selftest_wait_timeout(void* ws, qs_stream_t stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return QS_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<uint32_t*>(ws), 1u << 14);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}
