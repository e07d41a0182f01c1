// Routing: top-k per token, softmax over the selected logits, and a
// deterministic counting sort of the token slots by (expert, token).
//
// Pages: "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview,
// and "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
// section "NVFP4 and MXFP8 experts": each token is routed to 8 of 384
// experts, with no shared expert.
//
// Large batches: three kernels after two small memsets (token bitmaps to
// zero, every row of sorted_slots to -1):
//   1. route_topk_kernel  one warp per token, 8 tokens per CTA: top-k by k
//      warp-wide max rounds (ties to the lower index), the softmax, and
//      bit t of the expert's token bitmap set (atomicOr, order-independent).
//   2. route_scan_kernel  one CTA per expert: the exclusive prefix of popc
//      over its bitmap words (its slot count at the end); the last CTA to
//      finish scans the 128-padded counts into the expert offsets.
//   3. route_scatter_kernel  one thread per slot: row = offset[e] +
//      prefix[e][t/32] + (tokens before t in word t/32 that chose e).
// Small batches (route_small: up to 512 tokens) take two kernels and no
// memset: the top-k kernel without the bitmaps, then route_small_kernel, one
// CTA that builds the token bitmaps in shared memory and writes the counts,
// the padded offsets, the padding rows and the slot scatter; same results.
// Nothing depends on thread timing, so the result is deterministic.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "route_common.cuh"

namespace moe {

constexpr int kTopkWarps = 8;  // tokens per CTA of the top-k kernel

// Top-k of one token's logits (warp_topk_keys), then the softmax over the
// selected logits.  Every lane ends with the same sel_i; lane j < k holds w
// of rank j.
template <int NPL>
__device__ __forceinline__ void topk_token(const float* __restrict__ row, int E, int k, int lane, int* sel_i,
                                           float& w_lane) {
  uint32_t key[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? logit_key(__ldg(row + e)) : 0u;
  }
  const uint32_t my_key = warp_topk_keys<NPL>(key, k, lane, sel_i);
  w_lane = warp_topk_softmax(key_logit(my_key), k, lane);
}

// NPL = logits per lane (ceil(E / 32)); W = bitmap words per expert.
template <int NPL>
__global__ void __launch_bounds__(kTopkWarps * 32) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                     int k, int W, int32_t* __restrict__ topk_ids,
                                                                     float* __restrict__ topk_w,
                                                                     uint32_t* __restrict__ bitmap) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  int sel_i[8];
  float w;
  topk_token<NPL>(logits + static_cast<int64_t>(t) * E, E, k, lane, sel_i, w);
  int my_e = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (lane == j) my_e = sel_i[j];
  if (lane < k) {
    topk_ids[static_cast<int64_t>(t) * k + lane] = my_e;
    topk_w[static_cast<int64_t>(t) * k + lane] = w;
    if (bitmap != nullptr) atomicOr(&bitmap[static_cast<int64_t>(my_e) * W + (t >> 5)], 1u << (t & 31));
  }
}

constexpr int kScanThreads = 256;
constexpr int kScanWordsPerThread = 4;

// One CTA per expert: prefix[e][i] = sum of popc over words 0..i-1 of expert
// e's token bitmap (kScanWordsPerThread consecutive words per thread, one
// block-wide scan per 1024 words), and expert_counts[e].  The CTA that
// finishes last (a ticket counter, zeroed with the bitmaps) then scans the
// 128-padded counts of all experts into expert_offsets.  Which CTA that is
// depends on timing; what it computes does not.
__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(int E, int W, const uint32_t* __restrict__ bitmap,
                                                                  int32_t* __restrict__ prefix,
                                                                  int32_t* __restrict__ expert_counts,
                                                                  int32_t* __restrict__ expert_offsets,
                                                                  unsigned int* __restrict__ ticket) {
  __shared__ int32_t warp_sums[32];
  __shared__ int is_last;
  const int e = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const uint32_t* bm = bitmap + static_cast<int64_t>(e) * W;
  int32_t* pf = prefix + static_cast<int64_t>(e) * W;
  int32_t base = 0;
  for (int w0 = 0; w0 < W; w0 += kScanThreads * kScanWordsPerThread) {
    const int i0 = w0 + kScanWordsPerThread * threadIdx.x;
    int32_t c[kScanWordsPerThread];
    int32_t mine = 0;
#pragma unroll
    for (int j = 0; j < kScanWordsPerThread; ++j) {
      c[j] = (i0 + j < W) ? __popc(bm[i0 + j]) : 0;
      mine += c[j];
    }
    int32_t chunk_total = 0;
    int32_t run = base + block_exclusive_scan(mine, warp_sums, &chunk_total);
#pragma unroll
    for (int j = 0; j < kScanWordsPerThread; ++j) {
      if (i0 + j < W) pf[i0 + j] = run;
      run += c[j];
    }
    base += chunk_total;
    __syncthreads();  // warp_sums is reused by the next chunk's scan
  }
  if (threadIdx.x == 0) {
    expert_counts[e] = base;
    __threadfence();
    is_last = atomicAdd(ticket, 1u) == static_cast<unsigned int>(E - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // padded exclusive offsets over the experts, kScanWordsPerThread experts per thread
  const volatile int32_t* counts = expert_counts;
  int32_t padded[kScanWordsPerThread];
  int32_t mine = 0;
  const int e0 = kScanWordsPerThread * threadIdx.x;
#pragma unroll
  for (int j = 0; j < kScanWordsPerThread; ++j) {
    padded[j] = (e0 + j < E) ? (counts[e0 + j] + 127) / 128 * 128 : 0;
    mine += padded[j];
  }
  int32_t total = 0;
  int32_t run = block_exclusive_scan(mine, warp_sums, &total);
#pragma unroll
  for (int j = 0; j < kScanWordsPerThread; ++j) {
    if (e0 + j < E) expert_offsets[e0 + j] = run;
    run += padded[j];
  }
  if (threadIdx.x == 0) {
    expert_offsets[E] = total;
    *ticket = 0u;
  }
}

__global__ void route_scatter_kernel(int T, int E, int k, int W, const int32_t* __restrict__ topk_ids,
                                     const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ prefix,
                                     const int32_t* __restrict__ expert_offsets, int32_t* __restrict__ sorted_slots,
                                     int32_t* __restrict__ slot_to_row) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (s >= static_cast<int64_t>(T) * k) return;
  const int t = static_cast<int>(s / k);
  const int e = topk_ids[s];
  if (e < 0 || e >= E) return;  // only after a fused router gave up on a timeout (status word set)
  const int64_t wi = static_cast<int64_t>(e) * W + (t >> 5);
  const int rank = prefix[wi] + __popc(bitmap[wi] & ((1u << (t & 31)) - 1u));
  const int32_t row = expert_offsets[e] + rank;
  sorted_slots[row] = static_cast<int32_t>(s);
  slot_to_row[s] = row;
}

constexpr int kSmallThreads = 1024;

// Routing steps after the top-k for a small batch, in one CTA (E <= 1024,
// E * ceil(T / 32) <= kSmallWords): token bitmaps of every expert in shared
// memory, per-word prefix counts, the counts, the 128-padded offsets (one
// expert per thread, block scan), every row of sorted_slots set to -1, then
// the scatter.  Identical results to the scan / scatter kernels.
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(int T, int E, int k, int64_t R_max,
                                                                    const int32_t* __restrict__ topk_ids,
                                                                    int32_t* __restrict__ expert_counts,
                                                                    int32_t* __restrict__ expert_offsets,
                                                                    int32_t* __restrict__ sorted_slots,
                                                                    int32_t* __restrict__ slot_to_row) {
  extern __shared__ uint32_t sm_small[];
  __shared__ int32_t warp_sums[32];
  pdl_wait();
  pdl_trigger();
  small_route_block(T, E, k, R_max, topk_ids, expert_counts, expert_offsets, sorted_slots, slot_to_row, sm_small,
                    warp_sums);
}

bool route_small(int T, int E) {
  return T > 0 && T <= 512 && E <= kSmallThreads && static_cast<int64_t>(E) * ((T + 31) / 32) <= kSmallWords;
}

int64_t route_workspace_bytes(int E, int64_t T) {
  const int64_t W = (T + 31) / 32;
  return static_cast<int64_t>(E) * W * 8 + 256;  // bitmap words, ticket, their prefix counts
}

// Workspace: token bitmaps [E][W] words, a 16-byte ticket counter, prefix
// counts [E][W]; the bitmaps and the ticket are zeroed by route_prepare.
namespace {
unsigned int* ws_ticket(void* ws, int E, int W) {
  return reinterpret_cast<unsigned int*>(static_cast<uint32_t*>(ws) + static_cast<int64_t>(E) * W);
}
int32_t* ws_prefix(void* ws, int E, int W) {
  return reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + static_cast<int64_t>(E) * W * 4 + 16);
}
}  // namespace

cudaError_t route_prepare(int T, int E, int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                          int64_t R_max, void* workspace, cudaStream_t stream) {
  cudaError_t err = cudaSuccess;
  if (route_small(T, E)) return cudaSuccess;  // route_small_kernel writes everything itself
  if (R_max > 0) {
    err = cudaMemsetAsync(sorted_slots, 0xFF, static_cast<size_t>(R_max) * sizeof(int32_t), stream);
    if (err != cudaSuccess) return err;
  }
  if (T == 0) {
    err = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, stream);
    if (err != cudaSuccess) return err;
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), stream);
  }
  const int W = (T + 31) / 32;
  return cudaMemsetAsync(workspace, 0, static_cast<size_t>(E) * W * sizeof(uint32_t) + 16, stream);
}

cudaError_t route_finish(int T, int E, int k, const int32_t* topk_ids, int32_t* expert_counts,
                         int32_t* expert_offsets, int32_t* sorted_slots, int32_t* slot_to_row, int64_t R_max,
                         void* workspace, cudaStream_t stream) {
  const int W = (T + 31) / 32;
  if (route_small(T, E)) {
    const size_t smem = static_cast<size_t>(E) * W * 8 + static_cast<size_t>(E) * 4;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
      attr_err = cudaFuncSetAttribute(route_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(kSmallWords * 8 + kSmallThreads * 4));
    });
    if (attr_err != cudaSuccess) return attr_err;
    return launch_pdl(route_small_kernel, dim3(1), dim3(kSmallThreads), smem, stream, T, E, k, R_max, topk_ids,
                      expert_counts, expert_offsets, sorted_slots, slot_to_row);
  }
  const uint32_t* bitmap = static_cast<const uint32_t*>(workspace);
  int32_t* prefix = ws_prefix(workspace, E, W);
  cudaError_t err = launch_pdl(route_scan_kernel, dim3(E), dim3(kScanThreads), 0, stream, E, W, bitmap, prefix,
                               expert_counts, expert_offsets, ws_ticket(workspace, E, W));
  if (err != cudaSuccess) return err;
  const int64_t slots = static_cast<int64_t>(T) * k;
  return launch_pdl(route_scatter_kernel, dim3(static_cast<unsigned>((slots + 255) / 256)), dim3(256), 0, stream, T,
                    E, k, W, topk_ids, bitmap, static_cast<const int32_t*>(prefix),
                    static_cast<const int32_t*>(expert_offsets), sorted_slots, slot_to_row);
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                         int32_t* slot_to_row, int64_t R_max, void* workspace, cudaStream_t stream) {
  cudaError_t err = route_prepare(T, E, expert_counts, expert_offsets, sorted_slots, R_max, workspace, stream);
  if (err != cudaSuccess || T == 0) return err;
  const int W = (T + 31) / 32;
  uint32_t* bitmap = route_small(T, E) ? nullptr : static_cast<uint32_t*>(workspace);
  const int npl = (E + 31) / 32;
  const dim3 grid((T + kTopkWarps - 1) / kTopkWarps), block(kTopkWarps * 32);
  const float* lg = logits;
  if (npl <= 1)
    err = launch_pdl(route_topk_kernel<1>, grid, block, 0, stream, lg, T, E, k, W, topk_ids, topk_w, bitmap);
  else if (npl <= 4)
    err = launch_pdl(route_topk_kernel<4>, grid, block, 0, stream, lg, T, E, k, W, topk_ids, topk_w, bitmap);
  else if (npl <= 12)
    err = launch_pdl(route_topk_kernel<12>, grid, block, 0, stream, lg, T, E, k, W, topk_ids, topk_w, bitmap);
  else
    err = launch_pdl(route_topk_kernel<32>, grid, block, 0, stream, lg, T, E, k, W, topk_ids, topk_w, bitmap);
  if (err != cudaSuccess) return err;
  return route_finish(T, E, k, topk_ids, expert_counts, expert_offsets, sorted_slots, slot_to_row, R_max, workspace,
                      stream);
}

}  // namespace moe
