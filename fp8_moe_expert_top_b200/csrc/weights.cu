// Offline expert-weight quantization into the GEMM-ready packed layout.
//
// Pages: "thinkingmachines/Inkling-2-Small", section Overview (NVFP4 experts
// in layers 0-39, MXFP8 in layers 40-47) and "Thinking Machines releases
// Inkling 2 Small weights under Apache 2.0", section TL;DR (the 4-vs-6 block
// scale pick of the NVFP4 quantizer).  NVFP4 tensor scale per (expert,
// matrix): amax / 2688 (2688 = 6 * 448), 1 for an all-zero matrix.
//
// Four steps on the stream: zero the amax slots, reduce amax per matrix
// (atomicMax on the float bits, exact and order-independent for values >= 0),
// quantize every 64-element group, turn amax into the tensor scale.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {

// blockIdx.y = matrix (0 gate, 1 up, 2 down), blockIdx.z = expert in the slice
__global__ void __launch_bounds__(256) weight_amax_kernel(int64_t n_per_matrix, const float* __restrict__ w_gate,
                                                          const float* __restrict__ w_up,
                                                          const float* __restrict__ w_down,
                                                          float* __restrict__ amax_out) {
  const int m = blockIdx.y, e = blockIdx.z;
  const float* w = (m == 0 ? w_gate : (m == 1 ? w_up : w_down)) + static_cast<int64_t>(e) * n_per_matrix;
  float a = 0.0f;
  const int64_t n4 = n_per_matrix / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(w) + i);
    a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
    atomicMax(reinterpret_cast<unsigned int*>(amax_out + e * 3 + m), __float_as_uint(a));
  }
}

// One thread per 64-element group of one row.
template <int FMT>
__global__ void __launch_bounds__(256) weight_quant_kernel(int H, int I, const float* __restrict__ w_gate,
                                                           const float* __restrict__ w_up,
                                                           const float* __restrict__ w_down,
                                                           const float* __restrict__ amax, uint8_t* __restrict__ w13_codes,
                                                           uint8_t* __restrict__ w13_sf,
                                                           uint8_t* __restrict__ w2_codes,
                                                           uint8_t* __restrict__ w2_sf) {
  const int m = blockIdx.y, e = blockIdx.z;  // e: index inside the slice (pointers are already offset)
  const int64_t n_per_matrix = static_cast<int64_t>(I) * H;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= n_per_matrix / 64) return;
  const int K = (m == 2) ? I : H;
  const int G = K / 64;
  const int64_t src_row = gid / G;
  const int g = static_cast<int>(gid % G);
  const float* src = (m == 0 ? w_gate : (m == 1 ? w_up : w_down)) + static_cast<int64_t>(e) * n_per_matrix +
                     src_row * K + 64 * g;
  // destination row: gate/up interleaved in groups of 32 rows inside w13
  int64_t dst_row;
  uint8_t *codes, *sfbuf;
  int64_t rows_per_expert;
  if (m == 2) {
    dst_row = src_row;
    rows_per_expert = H;
    codes = w2_codes;
    sfbuf = w2_sf;
  } else {
    dst_row = 64 * (src_row / 32) + (m == 1 ? 32 : 0) + (src_row % 32);
    rows_per_expert = 2 * static_cast<int64_t>(I);
    codes = w13_codes;
    sfbuf = w13_sf;
  }
  const float4* src4 = reinterpret_cast<const float4*>(src);
  const int64_t kb = kb_padded(K, FMT == MOE_NVFP4 ? 4 : 8);
  uint8_t* ecodes = codes + static_cast<int64_t>(e) * rows_per_expert * kb;  // this expert's tiles
  if (FMT == MOE_NVFP4) {
    const float a = amax[e * 3 + m];
    const float s_g = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
    uint32_t sfw = 0;
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
      float f[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(src4 + 4 * b + i);
        f[4 * i] = v.x;
        f[4 * i + 1] = v.y;
        f[4 * i + 2] = v.z;
        f[4 * i + 3] = v.w;
      }
      const Nvfp4Block q = nvfp4_quantize16(f, s_g);
      sfw |= q.sf << (8 * b);
      *reinterpret_cast<uint2*>(ecodes + tile_offset(dst_row, 32 * g + 8 * b, kb, kWeightTileRows)) =
          make_uint2(static_cast<uint32_t>(q.codes), static_cast<uint32_t>(q.codes >> 32));
    }
    const int64_t nsf = K / 16;
    uint8_t* sfe = sfbuf + static_cast<int64_t>(e) * rows_per_expert * nsf;
    *reinterpret_cast<uint32_t*>(sfe + sf_offset(dst_row, 4 * g, nsf)) = sfw;
  } else {
    uint32_t sfw = 0;
#pragma unroll 1
    for (int b = 0; b < 2; ++b) {
      float f[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = __ldg(src4 + 8 * b + i);
        f[4 * i] = v.x;
        f[4 * i + 1] = v.y;
        f[4 * i + 2] = v.z;
        f[4 * i + 3] = v.w;
      }
      uint32_t w[8];
      sfw |= mxfp8_quantize32(f, w) << (8 * b);
      const int byte0 = 64 * g + 32 * b;
      *reinterpret_cast<uint4*>(ecodes + tile_offset(dst_row, byte0, kb, kWeightTileRows)) =
          make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(ecodes + tile_offset(dst_row, byte0 + 16, kb, kWeightTileRows)) =
          make_uint4(w[4], w[5], w[6], w[7]);
    }
    const int64_t nsf = K / 32;
    uint8_t* sfe = sfbuf + static_cast<int64_t>(e) * rows_per_expert * nsf;
    *reinterpret_cast<uint16_t*>(sfe + sf_offset(dst_row, 2 * g, nsf)) = static_cast<uint16_t>(sfw);
  }
}

__global__ void weight_scale_finalize_kernel(int n, int fmt, float* __restrict__ scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  if (fmt == MOE_NVFP4) {
    const float a = scales[i];
    scales[i] = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
  } else {
    scales[i] = 1.0f;
  }
}

cudaError_t launch_quantize_weights(int fmt, int E, int H, int I, int expert_begin, int expert_count,
                                    const float* w_gate, const float* w_up, const float* w_down, uint8_t* w13_codes,
                                    uint8_t* w13_sf, uint8_t* w2_codes, uint8_t* w2_sf, float* scales,
                                    cudaStream_t stream) {
  (void)E;
  if (expert_count == 0) return cudaSuccess;
  const int bits = (fmt == MOE_NVFP4) ? 4 : 8;
  const int sfvec = (fmt == MOE_NVFP4) ? 16 : 32;
  const int64_t rows13 = 2 * static_cast<int64_t>(I);
  // offset every output by the slice start so the kernels index experts 0..count-1
  uint8_t* c13 = w13_codes + static_cast<int64_t>(expert_begin) * rows13 * kb_padded(H, bits);
  uint8_t* s13 = w13_sf + static_cast<int64_t>(expert_begin) * rows13 * H / sfvec;
  uint8_t* c2 = w2_codes + static_cast<int64_t>(expert_begin) * H * kb_padded(I, bits);
  uint8_t* s2 = w2_sf + static_cast<int64_t>(expert_begin) * H * static_cast<int64_t>(I) / sfvec;
  float* sc = scales + static_cast<int64_t>(expert_begin) * 3;
  cudaError_t err = cudaMemsetAsync(sc, 0, sizeof(float) * 3 * expert_count, stream);
  if (err != cudaSuccess) return err;
  const int64_t n = static_cast<int64_t>(I) * H;
  if (fmt == MOE_NVFP4) {
    const int bx = static_cast<int>((n / 4 + 255) / 256 < 512 ? (n / 4 + 255) / 256 : 512);
    weight_amax_kernel<<<dim3(bx, 3, expert_count), 256, 0, stream>>>(n, w_gate, w_up, w_down, sc);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const dim3 grid(static_cast<unsigned>((n / 64 + 255) / 256), 3, expert_count);
  if (fmt == MOE_NVFP4)
    weight_quant_kernel<MOE_NVFP4><<<grid, 256, 0, stream>>>(H, I, w_gate, w_up, w_down, sc, c13, s13, c2, s2);
  else
    weight_quant_kernel<MOE_MXFP8><<<grid, 256, 0, stream>>>(H, I, w_gate, w_up, w_down, sc, c13, s13, c2, s2);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  weight_scale_finalize_kernel<<<(3 * expert_count + 255) / 256, 256, 0, stream>>>(3 * expert_count, fmt, sc);
  return cudaGetLastError();
}



// ---------------------------------------------------------------------------
// BF16 experts with LoRA adapters (pages "thinkingmachines/Inkling-2-Small",
// section Configurations, and "Thinking Machines releases Inkling 2 Small
// weights under Apache 2.0", section "LoRA and reinforcement learning":
// expert adapters need BF16 expert weights).  The bf16 weights are copied
// into the tiled layout with one extra 64-element K tile per row holding the
// adapter's B (gate rows: B_gate then zeros; up rows: zeros then B_up; down
// rows: B_down then zeros); the A matrices (gate and up stacked, down and
// zero rows) go to their own 64-row tiles.  Ranks below 32 are zero-padded.
// ---------------------------------------------------------------------------
namespace {

struct PackBf16Args {
  const __nv_bfloat16 *wg, *wu, *wd;  // [n][I][H], [n][I][H], [n][H][I]
  const __nv_bfloat16 *ag, *au, *ad;  // [n][r][H], [n][r][H], [n][r][I]; null: no adapters
  const __nv_bfloat16 *bg, *bu, *bd;  // [n][I][r], [n][I][r], [n][H][r]
  uint8_t *w13, *s13, *w2, *s2;       // outputs, already offset to the slice's first expert
  int H, I, r;
};

// Eight bf16 of row `row` of a [rows][r] adapter B matrix, elements j0 .. j0+7
// (zero past the rank).
__device__ __forceinline__ uint4 load_b8(const __nv_bfloat16* b, int64_t row, int r, int j0) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = j0 + 2 * i;
    const uint16_t lo = (j < r) ? __bfloat16_as_ushort(b[row * r + j]) : 0;
    const uint16_t hi = (j + 1 < r) ? __bfloat16_as_ushort(b[row * r + j + 1]) : 0;
    w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// blockIdx.y: 0 = w13 rows, 1 = w2 rows, 2 = A of gate / up, 3 = A of down;
// blockIdx.z = expert in the slice; one thread per 16-byte chunk of a row.
__global__ void __launch_bounds__(256) pack_bf16_kernel(const PackBf16Args a) {
  const int part = blockIdx.y, e = blockIdx.z;
  const int H = a.H, I = a.I, r = a.r;
  int rows, K, TR;
  int64_t kb;
  uint8_t* out;
  if (part == 0) {
    rows = 2 * I; K = H; kb = 2 * static_cast<int64_t>(H) + 128; TR = kWeightTileRows;
    out = a.w13 + static_cast<int64_t>(e) * rows * kb;
  } else if (part == 1) {
    rows = H; K = I; kb = 2 * static_cast<int64_t>(I) + 128; TR = kWeightTileRows;
    out = a.w2 + static_cast<int64_t>(e) * rows * kb;
  } else if (part == 2) {
    rows = 64; K = H; kb = 2 * static_cast<int64_t>(H); TR = 64;
    out = a.s13 + static_cast<int64_t>(e) * rows * kb;
  } else {
    rows = 64; K = I; kb = 2 * static_cast<int64_t>(I); TR = 64;
    out = a.s2 + static_cast<int64_t>(e) * rows * kb;
  }
  const int64_t chunks = kb / 16;
  const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= rows * chunks) return;
  const int row = static_cast<int>(id / chunks);
  const int j0 = static_cast<int>(id % chunks) * 8;  // first element of the chunk
  const bool lora = a.ag != nullptr;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (part == 0) {
    const bool up = (row & 63) >= 32;
    const int64_t ch = 32 * (row / 64) + (row & 31);
    const __nv_bfloat16* w = (up ? a.wu : a.wg) + static_cast<int64_t>(e) * I * H;
    if (j0 < K) {
      v = __ldg(reinterpret_cast<const uint4*>(w + ch * H + j0));
    } else if (lora) {
      const int jj = j0 - K;  // 0 .. 63: gate B in 0..31, up B in 32..63
      if (!up && jj < 32) v = load_b8(a.bg + static_cast<int64_t>(e) * I * r, ch, r, jj);
      if (up && jj >= 32) v = load_b8(a.bu + static_cast<int64_t>(e) * I * r, ch, r, jj - 32);
    }
  } else if (part == 1) {
    const __nv_bfloat16* w = a.wd + static_cast<int64_t>(e) * H * I;
    if (j0 < K) {
      v = __ldg(reinterpret_cast<const uint4*>(w + static_cast<int64_t>(row) * I + j0));
    } else if (lora && j0 - K < 32) {
      v = load_b8(a.bd + static_cast<int64_t>(e) * H * r, row, r, j0 - K);
    }
  } else if (lora) {
    const __nv_bfloat16* m = nullptr;
    int ar = row;
    if (part == 2) {
      m = (row < 32) ? a.ag : a.au;
      ar = row & 31;
    } else if (row < 32) {
      m = a.ad;
    }
    if (m != nullptr && ar < r)
      v = __ldg(reinterpret_cast<const uint4*>(m + (static_cast<int64_t>(e) * r + ar) * K + j0));
  }
  *reinterpret_cast<uint4*>(out + tile_offset(row, 2 * static_cast<int64_t>(j0), kb, TR)) = v;
}

__global__ void bf16_scales_kernel(int n, float scaling, float* __restrict__ scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 3 * n) scales[i] = (i % 3 == 0) ? scaling : 0.0f;
}

}  // namespace

cudaError_t launch_pack_bf16(int H, int I, int expert_begin, int expert_count, const void* w_gate, const void* w_up,
                             const void* w_down, const void* a_gate, const void* a_up, const void* a_down,
                             const void* b_gate, const void* b_up, const void* b_down, int rank, float scaling,
                             uint8_t* w13, uint8_t* s13, uint8_t* w2, uint8_t* s2, float* scales,
                             cudaStream_t stream) {
  if (expert_count == 0) return cudaSuccess;
  PackBf16Args a;
  a.wg = static_cast<const __nv_bfloat16*>(w_gate);
  a.wu = static_cast<const __nv_bfloat16*>(w_up);
  a.wd = static_cast<const __nv_bfloat16*>(w_down);
  a.ag = static_cast<const __nv_bfloat16*>(a_gate);
  a.au = static_cast<const __nv_bfloat16*>(a_up);
  a.ad = static_cast<const __nv_bfloat16*>(a_down);
  a.bg = static_cast<const __nv_bfloat16*>(b_gate);
  a.bu = static_cast<const __nv_bfloat16*>(b_up);
  a.bd = static_cast<const __nv_bfloat16*>(b_down);
  const int64_t kb13 = 2 * static_cast<int64_t>(H) + 128, kb2 = 2 * static_cast<int64_t>(I) + 128;
  a.w13 = w13 + static_cast<int64_t>(expert_begin) * 2 * I * kb13;
  a.s13 = s13 + static_cast<int64_t>(expert_begin) * 64 * 2 * static_cast<int64_t>(H);
  a.w2 = w2 + static_cast<int64_t>(expert_begin) * H * kb2;
  a.s2 = s2 + static_cast<int64_t>(expert_begin) * 64 * 2 * static_cast<int64_t>(I);
  a.H = H;
  a.I = I;
  a.r = rank;
  const int64_t most = std::max(2 * static_cast<int64_t>(I) * kb13, static_cast<int64_t>(H) * kb2) / 16;
  pack_bf16_kernel<<<dim3(static_cast<unsigned>((most + 255) / 256), 4, expert_count), 256, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  bf16_scales_kernel<<<(3 * expert_count + 255) / 256, 256, 0, stream>>>(
      expert_count, a.ag != nullptr ? scaling : 0.0f, scales + static_cast<int64_t>(expert_begin) * 3);
  return cudaGetLastError();
}

}  // namespace moe
