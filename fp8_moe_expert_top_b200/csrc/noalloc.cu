// Routing without a caller-provided workspace.
//
// moe_route_topk needs scratch device memory (per-expert token bitmaps and
// their prefix counts).  Some callers cannot hand it any: a plugin inside another runtime
// that only receives its input and output tensors, a real-time or embedded
// host whose device memory is planned once up front, or a caller that may not
// touch the allocator at that point.  moe_route_topk_noalloc serves them by
// using a fixed scratch array that is part of the loaded library image
// instead.  It runs exactly the kernels of moe_route_topk, so its results are
// the same bit for bit.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/moe_b200.h"
#include "kernels.cuh"

namespace {

// Largest routing scratch the no-allocation entry point can use.  The array
// lives in device memory of every GPU that loads the library, until exit.
constexpr int64_t kScratchBytes = int64_t(4) << 20;  // 4 MiB

__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of g_route_scratch on device `dev`, which must be the
// current device (looked up once per device; host code cannot use the
// symbol itself as a device pointer).
cudaError_t scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_route_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" MOE_API moe_status moe_route_topk_noalloc(const moe_config* cfg, int64_t T, const float* logits,
                                                     int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                                                     int32_t* expert_offsets, int32_t* sorted_slots,
                                                     int32_t* slot_to_row, void* stream) {
  moe_status s = moe_check_config(cfg);
  if (s != MOE_OK) return s;
  const int64_t need = moe_route_workspace_bytes(cfg, T);
  if (need < 0) return MOE_ERR_UNSUPPORTED;
  if (need > kScratchBytes) return MOE_ERR_WORKSPACE;  // more tokens x experts than the fixed scratch holds
  // The scratch address is per device: the work must go to the current
  // device.  A stream of another device is refused before anything is
  // enqueued (the legacy and per-thread default streams belong to the current
  // device).
  int dev = 0, stream_dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (stream != nullptr) {
    if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &stream_dev) != cudaSuccess) return MOE_ERR_INVALID_ARG;
    if (stream_dev != dev) return MOE_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // Every byte of scratch that the kernels read is written earlier in the
  // same call, so nothing has to be cleared between calls.
  return moe_route_topk(cfg, T, logits, topk_ids, topk_w, expert_counts, expert_offsets, sorted_slots, slot_to_row,
                        scratch, kScratchBytes, stream);
}
