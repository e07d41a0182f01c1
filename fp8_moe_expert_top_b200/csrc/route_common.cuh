// Routing pieces shared by the top-k kernel over given logits and the fused
// router (GEMM + top-k): the warp-wide top-k selection and the softmax's
// exponential.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

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

// A logit as an unsigned key with the same order (-0 taken as +0, so that the
// two compare equal like the floats do); 0 is below every logit's key and
// marks an expert that is not there.
__device__ __forceinline__ uint32_t logit_key(float v) {
  const uint32_t b = __float_as_uint(__fadd_rn(v, 0.0f));
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k (k <= 8) of one token whose logits are spread over a warp: lane l
// holds the keys of experts l, l + 32, ... (NPL of them).  Each lane keeps
// its best key not yet taken; a round takes the warp's largest key and, among
// the lanes holding it, the lowest expert index (two warp reductions), and
// only the winning lane looks for its next best.  Every lane ends with the
// same sel_i[0..k); lane j < k returns the key of rank j.
template <int NPL>
__device__ __forceinline__ uint32_t warp_topk_keys(const uint32_t* key, int k, int lane, int* sel_i) {
  uint32_t taken = 0u;
  // this lane's best: largest key, the lower expert among equal keys
  uint32_t head = 0u;
  int head_i = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (key[i] > head) {
      head = key[i];
      head_i = i;
    }
  }
  uint32_t my_key = 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, head);
    const uint32_t my_e = static_cast<uint32_t>(lane + 32 * head_i);
    const uint32_t win = __reduce_min_sync(0xFFFFFFFFu, head == m ? my_e : 0xFFFFFFFFu);
    if (lane == j) my_key = m;
    sel_i[j] = static_cast<int>(win);
    if (my_e == win) {
      taken |= 1u << head_i;
      head = 0u;
      head_i = 0;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if (!((taken >> i) & 1u) && key[i] > head) {
          head = key[i];
          head_i = i;
        }
      }
    }
  }
  return my_key;
}

// Softmax over the k selected logits, lane j holding the logit of rank j:
// e_j = exp(l_j - l_0), s = ((e_0 + e_1) + e_2) + ... in rank order, and lane
// j < k returns e_j / s.
__device__ __forceinline__ float warp_topk_softmax(float my_v, int k, int lane) {
  const float mx = __shfl_sync(0xFFFFFFFFu, my_v, 0);
  const float ex = (lane < k) ? exp_own(__fsub_rn(my_v, mx)) : 0.0f;
  float s = __shfl_sync(0xFFFFFFFFu, ex, 0);
#pragma unroll
  for (int j = 1; j < 8; ++j) {
    const float ej = __shfl_sync(0xFFFFFFFFu, ex, j);
    if (j < k) s = __fadd_rn(s, ej);
  }
  return __fdiv_rn(ex, s);
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

// The counting sort of a small batch by one CTA (blockDim.x <= 1024), from
// topk_ids [T][k]: every expert's token bitmap (E * ceil(T/32) words) and its
// prefix counts in shared memory (smem: 2 E ceil(T/32) + E words), the slot
// counts, the 128-padded offsets (exclusive scan in expert order), -1 in
// every row of sorted_slots, then the scatter: row = offset[e] + (tokens
// before t that chose e).  An expert index outside [0, E) (possible only if
// the kernel that wrote topk_ids gave up on a timeout) is skipped, so no
// access leaves the arrays.
__device__ __forceinline__ void small_route_block(int T, int E, int k, int64_t R_max,
                                                  const int32_t* __restrict__ topk_ids,
                                                  int32_t* __restrict__ expert_counts,
                                                  int32_t* __restrict__ expert_offsets,
                                                  int32_t* __restrict__ sorted_slots,
                                                  int32_t* __restrict__ slot_to_row, uint32_t* smem,
                                                  int32_t* warp_sums) {
  const int W = (T + 31) >> 5;
  uint32_t* bm = smem;                                    // [E][W] token bitmaps
  int32_t* pf = reinterpret_cast<int32_t*>(smem + E * W);  // [E][W] prefix counts
  int32_t* off = pf + E * W;                              // [E] padded offsets
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < E * W; i += nt) bm[i] = 0u;
  __syncthreads();
  const int S = T * k;
  for (int s = tid; s < S; s += nt) {
    const int t = s / k, e = topk_ids[s];
    if (e >= 0 && e < E) atomicOr(&bm[e * W + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  // experts [tid * per, (tid + 1) * per) per thread, so that the scan runs
  // in expert order
  const int per = (E + nt - 1) / nt;
  const int e_lo = min(E, tid * per), e_hi = min(E, e_lo + per);
  int32_t mine = 0;
  for (int e = e_lo; e < e_hi; ++e) {
    int32_t cnt = 0;
    for (int w = 0; w < W; ++w) {
      pf[e * W + w] = cnt;
      cnt += __popc(bm[e * W + w]);
    }
    expert_counts[e] = cnt;
    mine += (cnt + 127) / 128 * 128;
  }
  int32_t total = 0;
  int32_t run = block_exclusive_scan(mine, warp_sums, &total);
  for (int e = e_lo; e < e_hi; ++e) {
    expert_offsets[e] = run;
    off[e] = run;
    const int32_t cnt = pf[e * W + W - 1] + __popc(bm[e * W + W - 1]);
    run += (cnt + 127) / 128 * 128;
  }
  if (tid == 0) expert_offsets[E] = total;
  for (int64_t r = tid; r < R_max; r += nt) sorted_slots[r] = -1;
  __syncthreads();  // the padding marks land before the scatter overwrites the used rows
  for (int s = tid; s < S; s += nt) {
    const int t = s / k, e = topk_ids[s];
    if (e < 0 || e >= E) continue;
    const int i = e * W + (t >> 5);
    const int32_t row = off[e] + pf[i] + __popc(bm[i] & ((1u << (t & 31)) - 1u));
    sorted_slots[row] = s;
    slot_to_row[s] = row;
  }
}

}  // namespace moe
