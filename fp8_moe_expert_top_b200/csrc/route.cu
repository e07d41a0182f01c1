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
constexpr int kTopkWarps = 8;

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
    const float* row = logits + static_cast<int64_t>(t) * E;
    float v[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
    }
    uint32_t taken = 0u;
    float sel_v[8];
    int sel_i[8];
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
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
    // softmax over the selected logits, in rank order (every lane computes it)
    float ex[8];
    float s = 0.0f;
    const float m = sel_v[0];
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
      ex[j] = exp_own(__fsub_rn(sel_v[j], m));
      s = (j == 0) ? ex[0] : __fadd_rn(s, ex[j]);
    }
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
      if (lane == j) {
        topk_ids[static_cast<int64_t>(t) * k + j] = sel_i[j];
        topk_w[static_cast<int64_t>(t) * k + j] = __fdiv_rn(ex[j], s);
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
