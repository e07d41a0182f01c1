// Block quantizers shared by the weight quantizer, the permute-gather and
// the gate/up GEMM epilogue.
//
// NVFP4 ("Thinking Machines releases Inkling 2 Small weights under Apache
// 2.0", section TL;DR): each 16-element block's maximum is mapped to both 4
// and 6 and the candidate with the lower error is kept.  The error of a
// candidate is the sum of squared errors in the dequantized domain summed by
// the fixed pairwise tree ((d0+d1)+(d2+d3))+..., candidate 4 wins only when
// strictly lower (ties to 6).  Every operation below is one IEEE float32
// rounding (explicit _rn intrinsics, so nothing is contracted into an FMA),
// which makes the result a pure function of the inputs and bit-identical to
// any other implementation that performs the same operations.
//
// MXFP8 ("thinkingmachines/Inkling-2-Small", section Overview: MXFP8 experts
// in layers 40-47): 32-element blocks, E8M0 scale 2^(e-127) with
// e = clamp(floor(log2 amax) - 8 + 127, 0, 254) (OCP MX rule), E4M3 codes of
// x * 2^(127-e), round-to-nearest-even with saturation.
#pragma once

#include <cstdint>
#include <cuda_fp8.h>

namespace moe {

// E2M1 magnitude code of v >= 0, round to nearest, ties to the even code,
// saturating at 6.  The decision points are the midpoints between the eight
// magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}; the comparison (> or >=) at each
// midpoint sends a tie to the neighbour with a zero mantissa bit.
__device__ __forceinline__ uint32_t e2m1_mag_code(float v) {
  return static_cast<uint32_t>(v > 0.25f) + static_cast<uint32_t>(v >= 0.75f) +
         static_cast<uint32_t>(v > 1.25f) + static_cast<uint32_t>(v >= 1.75f) +
         static_cast<uint32_t>(v > 2.5f) + static_cast<uint32_t>(v >= 3.5f) + static_cast<uint32_t>(v > 5.0f);
}

// Magnitude of a 3-bit E2M1 code: twice the magnitudes {0,1,2,3,4,6,8,12}
// packed as nibbles, halved.
__device__ __forceinline__ float e2m1_mag_value(uint32_t c) {
  return static_cast<float>((0xC8643210u >> (4 * c)) & 0xFu) * 0.5f;
}

// E4M3 (FN) encode, round to nearest even, saturating to +-448.  A zero
// result is returned as the canonical +0 code.
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
  uint32_t c = static_cast<uint32_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
  return (c & 0x7Fu) ? c : 0u;
}

// E4M3 (FN) decode of a non-NaN code (exact).
__device__ __forceinline__ float e4m3_decode(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v = (e == 0) ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80u) ? -v : v;
}

struct Nvfp4Block {
  uint64_t codes;  // element i in bits [4i, 4i+4): byte j = elements 2j (low) and 2j+1 (high)
  uint32_t sf;     // E4M3 block-scale code
};

// Quantize one candidate: the block maximum a is mapped to c (4 or 6).
__device__ __forceinline__ float nvfp4_candidate(const float* x, float a, float s_g, float c, uint64_t& codes,
                                                 uint32_t& sf) {
  const float denom = __fmul_rn(c, s_g);
  const float ratio = __fdiv_rn(a, denom);
  sf = e4m3_encode(ratio);
  const float S = __fmul_rn(e4m3_decode(sf), s_g);
  float d2[16];
  codes = 0;
  if (S == 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) d2[i] = __fmul_rn(x[i], x[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float q = __fdiv_rn(fabsf(x[i]), S);
      const uint32_t m = e2m1_mag_code(q);
      const float r = __fmul_rn(e2m1_mag_value(m), S);
      const bool neg = x[i] < 0.0f;
      const uint32_t code = m | ((neg && m != 0u) ? 8u : 0u);
      codes |= static_cast<uint64_t>(code) << (4 * i);
      const float d = __fsub_rn(x[i], neg ? -r : r);
      d2[i] = __fmul_rn(d, d);
    }
  }
  // fixed pairwise tree
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int i = 0; i < w; ++i) d2[i] = __fadd_rn(d2[2 * i], d2[2 * i + 1]);
  }
  return d2[0];
}

// NVFP4 4-vs-6 quantization of 16 float32 values with tensor scale s_g > 0.
__device__ __forceinline__ Nvfp4Block nvfp4_quantize16(const float* x, float s_g) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  uint64_t c6, c4;
  uint32_t e6, e4;
  const float err6 = nvfp4_candidate(x, a, s_g, 6.0f, c6, e6);
  const float err4 = nvfp4_candidate(x, a, s_g, 4.0f, c4, e4);
  Nvfp4Block b;
  const bool four = err4 < err6;
  b.codes = four ? c4 : c6;
  b.sf = four ? e4 : e6;
  return b;
}

// MXFP8 quantization of 32 float32 values: codes (4 bytes per uint32, element
// i in byte i%4 of word i/4) and the E8M0 exponent.
__device__ __forceinline__ uint32_t mxfp8_quantize32(const float* x, uint32_t* words) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(x[i]));
  const uint32_t ef = (__float_as_uint(a) >> 23) & 0xFFu;  // biased exponent; 0 for zero / subnormal
  const uint32_t e = ef >= 8u ? ef - 8u : 0u;              // floor(log2 a) - 8 + 127, clamped at 0
  const float scale = __uint_as_float((254u - e) << 23);   // 2^(127 - e), e <= 246
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) word |= e4m3_encode(__fmul_rn(x[4 * w + b], scale)) << (8 * b);
    words[w] = word;
  }
  return e;
}

}  // namespace moe
