// Self-test of the failure-detection path: a wait that can never complete
// must give up after its limit and report through the status word, leaving
// the CUDA context usable.  Nothing here faults or traps the GPU.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe_b200.h"
#include "common.cuh"

namespace {

// One CTA: thread 0 initializes an mbarrier that expects one arrival and no
// thread ever arrives; every warp's lane 0 waits on it with the bounded wait
// the GEMM roles use.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    moe::mbar_init(&bar, 1);
    abort_flag = 0;
    moe::fence_mbar_init();
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    if (!moe::mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicOr(status, MOE_DEVICE_TIMEOUT_SELFTEST);
  }
  __syncthreads();
}

}  // namespace

extern "C" MOE_API moe_status moe_selftest_bounded_wait(uint32_t* status_word, int64_t limit_ns, void* stream) {
  if (status_word == nullptr) return MOE_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 5000000000ll) return MOE_ERR_INVALID_ARG;
  bounded_wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(status_word,
                                                                                static_cast<uint64_t>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
