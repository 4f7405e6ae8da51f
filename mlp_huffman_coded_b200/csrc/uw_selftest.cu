// Self-test of the bounded waits every kernel of this library relies on: a
// wait whose condition never comes true must give up after its limit, record
// UW_ERR_TIMEOUT in the workspace status word and return, leaving the CUDA
// context usable.  The conditions are an mbarrier phase nothing completes and
// a counter nothing increments, so the test needs no fault and no hang.
#include <cuda_runtime.h>

#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

// words[0], words[1]: 1 if the mbarrier / counter wait returned true (it
// must not); words[2]: the counter, zero.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, uint32_t* words, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool a = mbar_wait_for(&bar, 0, nullptr, status, limit_ns);
    const bool b = wait_count_at_least(words + 2, 1u, nullptr, status, limit_ns);
    words[0] = a ? 1u : 0u;
    words[1] = b ? 1u : 0u;
    mbar_arrive(&bar);  // complete the phase: nothing is left pending at exit
  }
}

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_selftest_bounded_wait(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                              void* stream) {
  if (!workspace || workspace_bytes < kWsHeader || !aligned16(workspace)) return UW_ERR_INVALID_ARG;
  if (limit_us == 0 || limit_us > 1000000) return UW_ERR_INVALID_ARG;
  DeviceInfo dev;
  uw_status st = device_info(&dev);
  if (st != UW_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* words = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + 64);
  if (cudaMemsetAsync(words, 0, 16, s) != cudaSuccess) return UW_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t*>(workspace), words,
                                                static_cast<uint64_t>(limit_us) * 1000ull);
  note_launch();
  return cuda_status(cudaGetLastError());
}
