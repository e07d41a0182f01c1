// Permute-gather with fused activation quantization, and the weighted
// un-permute / combine.
//
// Page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
// section "NVFP4 and MXFP8 experts": expert activations are quantized to the
// layer's weight format inside the kernel that produces them, with no
// separate quantization pass.  Here the producer of the GEMM1 operand is the
// permute-gather: each token row is read once, quantized once (NVFP4 4-vs-6
// or MXFP8) and written to each of its k expert rows.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {

// 16 bf16 -> float
__device__ __forceinline__ void load16_bf16(const __nv_bfloat16* p, float* f) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 u = __ldg(q + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
      f[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

// One thread per (token, G elements): G = 32 (two NVFP4 blocks or one MXFP8
// block) for large batches, G = 16 (one NVFP4 block) for small ones, where
// more threads in flight matter more than fewer, wider stores.  The elements
// are read once, quantized once, and their codes and scale byte(s) are
// written to each of the token's k rows.  Four CTAs per SM (a 64-register
// cap): the quantizer's dependent chains gain more from the extra warps than
// they lose to a few spilled bytes (measured 4% faster than three CTAs at 79
// registers).
template <int FMT, int G>
__global__ void __launch_bounds__(256, 4) permute_kernel(int T, int H, int k, const __nv_bfloat16* __restrict__ x,
                                                      const float* __restrict__ act_scale,
                                                      const int32_t* __restrict__ slot_to_row,
                                                      uint8_t* __restrict__ a_codes, uint8_t* __restrict__ a_sf) {
  static_assert(G == 32 || (G == 16 && FMT == MOE_NVFP4), "group size");
  constexpr int kSfVec = (FMT == MOE_NVFP4) ? 16 : 32;
  const int nsf = H / kSfVec;
  const int ng = H / G;  // groups per token
  const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (id >= static_cast<int64_t>(T) * ng) return;
  const int t = static_cast<int>(id / ng);
  const int g = static_cast<int>(id % ng);
  float f[G];
#pragma unroll
  for (int i = 0; i < G / 16; ++i) load16_bf16(x + static_cast<int64_t>(t) * H + G * g + 16 * i, f + 16 * i);
  const int64_t kb = kb_padded(H, FMT == MOE_NVFP4 ? 4 : 8);
  if (FMT == MOE_NVFP4 && G == 16) {
    const Nvfp4Block q = nvfp4_quantize16(f, make_nvfp4_scale(__ldg(act_scale)));
    const uint2 c = make_uint2(static_cast<uint32_t>(q.codes), static_cast<uint32_t>(q.codes >> 32));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      const int64_t r = __ldg(slot_to_row + static_cast<int64_t>(t) * k + j);
      *reinterpret_cast<uint2*>(a_codes + tile_offset(r, 8 * g, kb, kActTileRows)) = c;
      a_sf[sf_offset(r, g, nsf)] = static_cast<uint8_t>(q.sf);
    }
  } else if (FMT == MOE_NVFP4) {
    const Nvfp4Scale s_x = make_nvfp4_scale(__ldg(act_scale));
    // both blocks through one copy of the quantizer's code: the kernel is
    // bound by its instruction stream, and two inlined copies measured 6-10%
    // slower (instruction-cache misses)
    Nvfp4Block q0, q1;
#pragma unroll 1
    for (int b = 0; b < 2; ++b) {
      float blk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) blk[i] = b ? f[16 + i] : f[i];
      const Nvfp4Block q = nvfp4_quantize16(blk, s_x);
      if (b == 0) q0 = q;
      else q1 = q;
    }
    const uint4 c = make_uint4(static_cast<uint32_t>(q0.codes), static_cast<uint32_t>(q0.codes >> 32),
                               static_cast<uint32_t>(q1.codes), static_cast<uint32_t>(q1.codes >> 32));
    const uint16_t sf = static_cast<uint16_t>(q0.sf | (q1.sf << 8));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      const int64_t r = __ldg(slot_to_row + static_cast<int64_t>(t) * k + j);
      *reinterpret_cast<uint4*>(a_codes + tile_offset(r, 16 * g, kb, kActTileRows)) = c;
      *reinterpret_cast<uint16_t*>(a_sf + sf_offset(r, 2 * g, nsf)) = sf;  // blocks 2g, 2g + 1: adjacent bytes
    }
  } else {
    uint32_t w[8];
    const uint32_t e = mxfp8_quantize32(f, w);
    const bool wide = (reinterpret_cast<uintptr_t>(a_codes) & 31u) == 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      const int64_t r = __ldg(slot_to_row + static_cast<int64_t>(t) * k + j);
      if (wide) {
        // the block's 32 code bytes as one store (one aligned slot under the swizzle)
        const int64_t o0 = tile_offset(r, 32 * g, kb, kActTileRows);
        const bool swap = ((r % kActTileRows) & 1) != 0;
        const uint32_t v[8] = {swap ? w[4] : w[0], swap ? w[5] : w[1], swap ? w[6] : w[2], swap ? w[7] : w[3],
                               swap ? w[0] : w[4], swap ? w[1] : w[5], swap ? w[2] : w[6], swap ? w[3] : w[7]};
        st_global_v8(a_codes + (swap ? o0 - 16 : o0), v);
      } else {
        *reinterpret_cast<uint4*>(a_codes + tile_offset(r, 32 * g, kb, kActTileRows)) =
            make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(a_codes + tile_offset(r, 32 * g + 16, kb, kActTileRows)) =
            make_uint4(w[4], w[5], w[6], w[7]);
      }
      a_sf[sf_offset(r, g, nsf)] = static_cast<uint8_t>(e);
    }
  }
}

// BF16 experts: no quantization; one thread per (token, 16 bytes of x) copies
// them into each of the token's k rows (tiled, with the adapter K tile after
// the d_model elements left to the adapter shrink).
__global__ void __launch_bounds__(256) permute_bf16_kernel(int T, int H, int k, const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ slot_to_row,
                                                           uint8_t* __restrict__ a_codes) {
  const int chunks = H / 8;
  const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (id >= static_cast<int64_t>(T) * chunks) return;
  const int t = static_cast<int>(id / chunks);
  const int c = static_cast<int>(id % chunks);
  const uint4 v = __ldg(x + id);
  const int64_t kb = 2 * static_cast<int64_t>(H) + 128;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    const int64_t r = __ldg(slot_to_row + static_cast<int64_t>(t) * k + j);
    *reinterpret_cast<uint4*>(a_codes + tile_offset(r, 16 * static_cast<int64_t>(c), kb, kActTileRows)) = v;
  }
}

cudaError_t launch_permute(int fmt, int T, int H, int k, const void* x, const float* act_scale,
                           const int32_t* slot_to_row, uint8_t* a_codes, uint8_t* a_sf, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (fmt == MOE_BF16) {
    const int64_t n = static_cast<int64_t>(T) * (H / 8);
    return launch_pdl(permute_bf16_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, stream, T, H,
                      k, static_cast<const uint4*>(x), slot_to_row, a_codes);
  }
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const dim3 block(256);
  // small batches (fewer 32-element groups than 256 per SM): one 16-element
  // NVFP4 block per thread doubles the threads in flight
  const bool small = fmt == MOE_NVFP4 && static_cast<int64_t>(T) * (H / 32) < 148 * 256;
  const int G = small ? 16 : 32;
  const dim3 grid(static_cast<unsigned>((static_cast<int64_t>(T) * (H / G) + 255) / 256));
  if (fmt == MOE_NVFP4) {
    if (small)
      return launch_pdl(permute_kernel<MOE_NVFP4, 16>, grid, block, 0, stream, T, H, k, xb, act_scale, slot_to_row,
                        a_codes, a_sf);
    return launch_pdl(permute_kernel<MOE_NVFP4, 32>, grid, block, 0, stream, T, H, k, xb, act_scale, slot_to_row,
                      a_codes, a_sf);
  }
  return launch_pdl(permute_kernel<MOE_MXFP8, 32>, grid, block, 0, stream, T, H, k, xb, act_scale, slot_to_row,
                    a_codes, a_sf);
}

// y[t] = sum_j w[t][j] * out[row(t, j)], float32 in rank order, then bf16.
// One CTA per token, one thread per 8 consecutive channels (a block of
// min(H / 8, 1024) threads, looping when H > 8192): the thread's k row loads
// are all issued before the arithmetic.
__global__ void __launch_bounds__(1024) combine_kernel(int H, int k, const __nv_bfloat16* __restrict__ down_out,
                                                       const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ slot_to_row,
                                                       __nv_bfloat16* __restrict__ y) {
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  float w[8];
  int64_t rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    w[j] = (j < k) ? __ldg(topk_w + static_cast<int64_t>(t) * k + j) : 0.0f;
    rows[j] = (j < k) ? __ldg(slot_to_row + static_cast<int64_t>(t) * k + j) : 0;
  }
  for (int c8 = threadIdx.x; c8 < H / 8; c8 += blockDim.x) {
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      u[j] = (j < k) ? __ldg(reinterpret_cast<const uint4*>(down_out + rows[j] * H) + c8) : make_uint4(0u, 0u, 0u, 0u);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      const uint32_t q[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w[j], __uint_as_float(q[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w[j], __uint_as_float(q[i] & 0xFFFF0000u)));
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    reinterpret_cast<uint4*>(y + static_cast<int64_t>(t) * H)[c8] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_combine(int T, int H, int k, const void* down_out, const float* topk_w,
                           const int32_t* slot_to_row, void* y, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int threads = std::min(1024, (H / 8 + 31) / 32 * 32);
  return launch_pdl(combine_kernel, dim3(T), dim3(static_cast<unsigned>(threads)), 0, stream, H, k,
                    static_cast<const __nv_bfloat16*>(down_out), topk_w, slot_to_row, static_cast<__nv_bfloat16*>(y));
}

}  // namespace moe
