// Routing: top-k per token, softmax over the selected logits, and a
// deterministic counting sort of the token slots by (expert, token).
//
// Pages: "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview,
// and "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
// section "NVFP4 and MXFP8 experts": each token is routed to 8 of 384
// experts, with no shared expert.
//
// Three kernels:
//   1. route_topk_kernel  one warp per token, 128 tokens per CTA: top-k by k
//      warp-wide arg-max rounds (ties to the lower index), the softmax, and a
//      per-CTA bitmap of which of its tokens chose each expert.
//   2. route_scan_kernel  one CTA: per-expert totals, the per-chunk exclusive
//      bases, and the padded expert offsets.
//   3. route_scatter_kernel  one thread per slot: row = offset[e] +
//      base[chunk][e] + (tokens of the chunk before t that chose e), counted
//      with popc on the bitmap.  Nothing depends on thread timing.
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// exp(x) for x <= 0 by Cody-Waite reduction and a degree-7 Taylor series,
// one float32 rounding per operation (see the header for the definition).
__device__ __forceinline__ float exp_own(float x) {
  const float kLog2e = 0x1.715476p+0f;      // log2(e) rounded to float32
  const float kLn2Hi = 0x1.62e4p-1f;        // 0.693145751953125 (16 significant bits)
  const float kLn2Lo = 0x1.7f7d1cp-20f;     // ln(2) - kLn2Hi rounded to float32
  // 1/i! rounded to float32, i = 0..7
  const float c0 = 1.0f, c1 = 1.0f, c2 = 0.5f, c3 = 0x1.555556p-3f, c4 = 0x1.555556p-5f,
              c5 = 0x1.111112p-7f, c6 = 0x1.6c16c2p-10f, c7 = 0x1.a01a02p-13f;
  if (x < -80.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, kLog2e));
  float r = __fsub_rn(x, __fmul_rn(n, kLn2Hi));
  r = __fsub_rn(r, __fmul_rn(n, kLn2Lo));
  float p = c7;
  p = __fadd_rn(__fmul_rn(p, r), c6);
  p = __fadd_rn(__fmul_rn(p, r), c5);
  p = __fadd_rn(__fmul_rn(p, r), c4);
  p = __fadd_rn(__fmul_rn(p, r), c3);
  p = __fadd_rn(__fmul_rn(p, r), c2);
  p = __fadd_rn(__fmul_rn(p, r), c1);
  p = __fadd_rn(__fmul_rn(p, r), c0);
  const float two_n = __uint_as_float(static_cast<uint32_t>(static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

constexpr int kChunk = 128;       // tokens per CTA in the top-k kernel
constexpr int kTopkWarps = 32;
constexpr int kSmallT = 1024;     // batches up to this size take the one-CTA path

// Top-k of one token's logits by k warp-wide arg-max rounds, then the softmax.
// Every lane ends with the same sel_i / w for j < k.
template <int NPL>
__device__ __forceinline__ void topk_token(const float* __restrict__ row, int E, int k, int lane, int* sel_i,
                                           float* w) {
  float v[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
  }
  uint32_t taken = 0u;
  float sel_v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      // strict '>' keeps the lower index among equal values of this lane
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || bi == 0x7FFFFFFF)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
      if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel_v[j] = bv;
    sel_i[j] = bi;
  }
  // softmax over the selected logits, in rank order
  float ex[8];
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    ex[j] = exp_own(__fsub_rn(sel_v[j], sel_v[0]));
    s = (j == 0) ? ex[0] : __fadd_rn(s, ex[j]);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    w[j] = __fdiv_rn(ex[j], s);
  }
}

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t ws = (lane < static_cast<int>(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, ws, off);
      if (lane >= off) ws += o;
    }
    warp_sums[lane] = ws;
  }
  __syncthreads();
  *total = warp_sums[(blockDim.x >> 5) - 1];
  return incl - v + (warp > 0 ? warp_sums[warp - 1] : 0);
}

// The whole routing step for T <= kSmallT in one CTA of 1024 threads: no
// workspace, no memset.  Token bitmaps per expert live in shared memory
// ([E][W] words, W = ceil(T / 32)), so slot ranks are popc counts and do not
// depend on thread timing.
template <int NPL>
__global__ void __launch_bounds__(1024) route_small_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                           int R_max, int32_t* __restrict__ topk_ids,
                                                           float* __restrict__ topk_w,
                                                           int32_t* __restrict__ expert_counts,
                                                           int32_t* __restrict__ expert_offsets,
                                                           int32_t* __restrict__ sorted_slots,
                                                           int32_t* __restrict__ slot_to_row) {
  extern __shared__ uint32_t sm[];
  const int W = (T + 31) / 32;
  uint32_t* bitmap = sm;                                   // [E][W]
  int32_t* s_off = reinterpret_cast<int32_t*>(sm + E * W);  // [E + 1]
  __shared__ int32_t warp_sums[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) bitmap[i] = 0u;
  __syncthreads();
  for (int t = warp; t < T; t += 32) {
    int sel_i[8];
    float w[8];
    topk_token<NPL>(logits + static_cast<int64_t>(t) * E, E, k, lane, sel_i, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      if (lane == j) {
        topk_ids[static_cast<int64_t>(t) * k + j] = sel_i[j];
        topk_w[static_cast<int64_t>(t) * k + j] = w[j];
        atomicOr(&bitmap[sel_i[j] * W + (t >> 5)], 1u << (t & 31));
      }
    }
  }
  __syncthreads();
  int32_t cnt = 0;
  const int e = threadIdx.x;
  if (e < E)
    for (int i = 0; i < W; ++i) cnt += __popc(bitmap[e * W + i]);
  const int32_t padded = ((cnt + 127) / 128) * 128;
  int32_t total = 0;
  const int32_t off = block_exclusive_scan(e < E ? padded : 0, warp_sums, &total);
  if (e < E) {
    s_off[e] = off;
    expert_counts[e] = cnt;
    expert_offsets[e] = off;
  }
  if (threadIdx.x == 0) {
    s_off[E] = total;
    expert_offsets[E] = total;
  }
  // every row starts as padding (coalesced), then the slots overwrite theirs
  for (int r = threadIdx.x; r < R_max; r += blockDim.x) sorted_slots[r] = -1;
  __syncthreads();
  for (int s = threadIdx.x; s < T * k; s += blockDim.x) {
    const int t = s / k;
    const int ex = topk_ids[s];
    const uint32_t* bm = bitmap + ex * W;
    int rank = __popc(bm[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int i = 0; i < (t >> 5); ++i) rank += __popc(bm[i]);
    const int32_t row = s_off[ex] + rank;
    sorted_slots[row] = s;
    slot_to_row[s] = row;
  }
}

// NPL = logits per lane (ceil(E / 32)).
template <int NPL>
__global__ void __launch_bounds__(kTopkWarps * 32) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                     int k, int32_t* __restrict__ topk_ids,
                                                                     float* __restrict__ topk_w,
                                                                     uint32_t* __restrict__ ws_bitmap,
                                                                     int32_t* __restrict__ ws_counts) {
  extern __shared__ uint32_t bitmap[];  // [E][4]: bit tl of word tl/32 = token tl of this chunk chose e
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  for (int i = threadIdx.x; i < E * 4; i += blockDim.x) bitmap[i] = 0u;
  __syncthreads();

  for (int tl = warp; tl < kChunk; tl += kTopkWarps) {
    const int t = chunk * kChunk + tl;
    if (t >= T) break;
    int sel_i[8];
    float w[8];
    topk_token<NPL>(logits + static_cast<int64_t>(t) * E, E, k, lane, sel_i, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      if (lane == j) {
        topk_ids[static_cast<int64_t>(t) * k + j] = sel_i[j];
        topk_w[static_cast<int64_t>(t) * k + j] = w[j];
        atomicOr(&bitmap[sel_i[j] * 4 + (tl >> 5)], 1u << (tl & 31));
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t b = bitmap[e * 4 + w];
      ws_bitmap[(static_cast<int64_t>(chunk) * E + e) * 4 + w] = b;
      c += __popc(b);
    }
    ws_counts[static_cast<int64_t>(chunk) * E + e] = static_cast<int32_t>(c);
  }
}

// One CTA of 1024 threads (E <= 1024).
__global__ void __launch_bounds__(1024) route_scan_kernel(int E, int nchunks, int32_t* __restrict__ ws_counts,
                                                           int32_t* __restrict__ expert_counts,
                                                           int32_t* __restrict__ expert_offsets) {
  __shared__ int32_t warp_sums[32];
  const int e = threadIdx.x;
  int32_t total = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int64_t idx = static_cast<int64_t>(c) * E + e;
      const int32_t cnt = ws_counts[idx];
      ws_counts[idx] = total;  // exclusive base of this chunk for expert e
      total += cnt;
    }
    expert_counts[e] = total;
  }
  const int32_t padded = (e < E) ? ((total + 127) / 128) * 128 : 0;
  // block-wide exclusive scan of padded
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = padded;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t ws = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, ws, off);
      if (lane >= off) ws += o;
    }
    warp_sums[lane] = ws;  // inclusive over warps
  }
  __syncthreads();
  const int32_t excl = incl - padded + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e < E) expert_offsets[e] = excl;
  if (e == E - 1) expert_offsets[E] = excl + padded;
}

__global__ void route_scatter_kernel(int T, int E, int k, const int32_t* __restrict__ topk_ids,
                                     const uint32_t* __restrict__ ws_bitmap, const int32_t* __restrict__ ws_base,
                                     const int32_t* __restrict__ expert_offsets, int32_t* __restrict__ sorted_slots,
                                     int32_t* __restrict__ slot_to_row) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (s >= static_cast<int64_t>(T) * k) return;
  const int t = static_cast<int>(s / k);
  const int e = topk_ids[s];
  const int chunk = t / kChunk, tl = t % kChunk;
  const uint32_t* bm = ws_bitmap + (static_cast<int64_t>(chunk) * E + e) * 4;
  int rank = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t b = bm[w];
    if (w < (tl >> 5)) rank += __popc(b);
    else if (w == (tl >> 5)) rank += __popc(b & ((1u << (tl & 31)) - 1u));
  }
  const int32_t row = expert_offsets[e] + ws_base[static_cast<int64_t>(chunk) * E + e] + rank;
  sorted_slots[row] = static_cast<int32_t>(s);
  slot_to_row[s] = row;
}

int64_t route_workspace_bytes(int E, int64_t T) {
  const int64_t nchunks = (T + kChunk - 1) / kChunk;
  return nchunks * E * (16 + 4) + 256;
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                         int32_t* slot_to_row, int64_t R_max, void* workspace, cudaStream_t stream) {
  const int npl_small = (E + 31) / 32;
  if (T > 0 && T <= kSmallT) {
    const int W = (T + 31) / 32;
    const size_t smem = static_cast<size_t>(E) * W * 4 + (static_cast<size_t>(E) + 1) * 4;
    static bool configured[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !configured[dev]) {
      const int max_smem = 1024 * 32 * 4 + (2 * 1024 + 1) * 4;
      cudaFuncSetAttribute(route_small_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      cudaFuncSetAttribute(route_small_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      cudaFuncSetAttribute(route_small_kernel<12>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      cudaFuncSetAttribute(route_small_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      if (dev < 64) configured[dev] = true;
    }
    const int R = static_cast<int>(R_max);
    if (npl_small <= 1)
      route_small_kernel<1><<<1, 1024, smem, stream>>>(logits, T, E, k, R, topk_ids, topk_w, expert_counts,
                                                        expert_offsets, sorted_slots, slot_to_row);
    else if (npl_small <= 4)
      route_small_kernel<4><<<1, 1024, smem, stream>>>(logits, T, E, k, R, topk_ids, topk_w, expert_counts,
                                                        expert_offsets, sorted_slots, slot_to_row);
    else if (npl_small <= 12)
      route_small_kernel<12><<<1, 1024, smem, stream>>>(logits, T, E, k, R, topk_ids, topk_w, expert_counts,
                                                         expert_offsets, sorted_slots, slot_to_row);
    else
      route_small_kernel<32><<<1, 1024, smem, stream>>>(logits, T, E, k, R, topk_ids, topk_w, expert_counts,
                                                         expert_offsets, sorted_slots, slot_to_row);
    return cudaGetLastError();
  }
  const int nchunks = (T + kChunk - 1) / kChunk;
  uint32_t* ws_bitmap = static_cast<uint32_t*>(workspace);
  int32_t* ws_counts = reinterpret_cast<int32_t*>(ws_bitmap + static_cast<int64_t>(nchunks) * E * 4);
  cudaError_t err = cudaMemsetAsync(sorted_slots, 0xFF, static_cast<size_t>(R_max) * sizeof(int32_t), stream);
  if (err != cudaSuccess) return err;
  if (T == 0) {
    err = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, stream);
    if (err != cudaSuccess) return err;
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), stream);
  }
  const int npl = (E + 31) / 32;
  const size_t smem = static_cast<size_t>(E) * 16;
  const dim3 grid(nchunks), block(kTopkWarps * 32);
  if (npl <= 1)
    route_topk_kernel<1><<<grid, block, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, ws_bitmap, ws_counts);
  else if (npl <= 4)
    route_topk_kernel<4><<<grid, block, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, ws_bitmap, ws_counts);
  else if (npl <= 12)
    route_topk_kernel<12><<<grid, block, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, ws_bitmap, ws_counts);
  else
    route_topk_kernel<32><<<grid, block, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, ws_bitmap, ws_counts);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  route_scan_kernel<<<1, 1024, 0, stream>>>(E, nchunks, ws_counts, expert_counts, expert_offsets);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t slots = static_cast<int64_t>(T) * k;
  route_scatter_kernel<<<static_cast<unsigned>((slots + 255) / 256), 256, 0, stream>>>(
      T, E, k, topk_ids, ws_bitmap, ws_counts, expert_offsets, sorted_slots, slot_to_row);
  return cudaGetLastError();
}

}  // namespace moe
