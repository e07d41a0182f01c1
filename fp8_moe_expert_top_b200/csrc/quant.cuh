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
#include <cuda_fp16.h>
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

// Hardware round-to-nearest-even conversions of two floats at once (lo goes
// to the low nibble / byte).
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Relative width of the bracket around an approximate quotient.  The
// approximation |x| * RN(1/S) is within 2^-23 (relative) of the exact
// quotient, so the exact quotient and its float32 rounding both lie strictly
// inside [q(1 - 2^-21), q(1 + 2^-21)].  When both ends of the bracket encode
// to the same code, so does RN(|x| / S) (the encoders are monotone); only
// otherwise is the exact division needed.  The results are therefore those
// of the plain definition, bit for bit.
constexpr float kBracketLo = 1.0f - 0x1p-21f;
constexpr float kBracketHi = 1.0f + 0x1p-21f;

// Exact slow paths, kept out of line so the common path stays small.
static __device__ __noinline__ uint32_t e2m1_code_exact(float num, float den) {
  return e2m1_mag_code(__fdiv_rn(num, den));
}
static __device__ __noinline__ uint32_t e4m3_code_exact(float num, float den) {
  return e4m3_encode(__fdiv_rn(num, den));
}

// E4M3 code of RN(num / den), num >= 0, den > 0, given rden = RN(1 / den).
__device__ __forceinline__ uint32_t e4m3_code_of_quotient_r(float num, float den, float rden) {
  if (num == 0.0f) return 0u;
  const float q = __fmul_rn(num, rden);
  const uint32_t pair = cvt_e4m3x2(__fmul_rn(q, kBracketLo), __fmul_rn(q, kBracketHi));
  const uint32_t lo = pair & 0xFFu, hi = pair >> 8;
  if (lo == hi) return lo;
  return e4m3_code_exact(num, den);
}
// E4M3 code of RN(num / den), num >= 0, den > 0.
__device__ __forceinline__ uint32_t e4m3_code_of_quotient(float num, float den) {
  return e4m3_code_of_quotient_r(num, den, __frcp_rn(den));
}

// Two E2M1 codes (element 2j in the low nibble) decoded to float (exact).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t pair) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t, u;\n\tmov.b16 {t, u}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2)
      : "h"(static_cast<uint16_t>(pair)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Per-thread constants of a tensor scale s_g: the reciprocals of both
// candidates' scale denominators RN(c s_g), c = 6 and 4.
struct Nvfp4Scale {
  float s_g, rd6, rd4;
};
__device__ __forceinline__ Nvfp4Scale make_nvfp4_scale(float s_g) {
  Nvfp4Scale t;
  t.s_g = s_g;
  t.rd6 = __frcp_rn(__fmul_rn(6.0f, s_g));
  t.rd4 = __frcp_rn(__fmul_rn(4.0f, s_g));
  return t;
}

// One candidate of the 4-vs-6 search on magnitudes ax[16] (block maximum a
// mapped to c).  Returns the squared error; mags receives the 3-bit
// magnitude codes (element i in bits [4i, 4i+4)), sf the scale code.
// Uses |x - dec(q)S| = ||x| - |dec(q)|S|, which holds bit for bit because
// rounding is symmetric in sign.
__device__ __forceinline__ float nvfp4_candidate(const float* ax, float a, float s_g, float c, uint64_t& mags,
                                                 uint32_t& sf) {
  sf = e4m3_code_of_quotient(a, __fmul_rn(c, s_g));
  const float S = __fmul_rn(e4m3_decode(sf), s_g);
  float d2[16];
  mags = 0;
  if (S == 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) d2[i] = __fmul_rn(ax[i], ax[i]);
  } else if (S >= 0x1p-100f) {
    const float rS = __frcp_rn(S);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      // both ends of both elements' brackets, two elements per conversion
      const float q0 = __fmul_rn(ax[i], rS), q1 = __fmul_rn(ax[i + 1], rS);
      const uint32_t lo = cvt_e2m1x2(__fmul_rn(q0, kBracketLo), __fmul_rn(q1, kBracketLo));
      const uint32_t hi = cvt_e2m1x2(__fmul_rn(q0, kBracketHi), __fmul_rn(q1, kBracketHi));
      uint32_t p = lo & 0x77u;
      if (lo != hi) {  // an end differs: settle that element by the exact division
        const uint32_t m0 = ((lo ^ hi) & 0x7u) ? e2m1_code_exact(ax[i], S) : (lo & 0x7u);
        const uint32_t m1 = ((lo ^ hi) & 0x70u) ? e2m1_code_exact(ax[i + 1], S) : ((lo >> 4) & 0x7u);
        p = m0 | (m1 << 4);
      }
      mags |= static_cast<uint64_t>(p) << (4 * i);
      const float2 v = e2m1x2_decode(p);
      const float d0 = __fsub_rn(ax[i], __fmul_rn(v.x, S));
      const float d1 = __fsub_rn(ax[i + 1], __fmul_rn(v.y, S));
      d2[i] = __fmul_rn(d0, d0);
      d2[i + 1] = __fmul_rn(d1, d1);
    }
  } else {  // tiny scales: exact division throughout
    // unrolled like the paths above: a runtime index into ax / d2 would put
    // both arrays in local memory for every call, not only for this path
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t m = e2m1_code_exact(ax[i], S);
      mags |= static_cast<uint64_t>(m) << (4 * i);
      const float d = __fsub_rn(ax[i], __fmul_rn(e2m1_mag_value(m), S));
      d2[i] = __fmul_rn(d, d);
    }
  }
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int i = 0; i < w; ++i) d2[i] = __fadd_rn(d2[2 * i], d2[2 * i + 1]);
  }
  return d2[0];
}

// One candidate with a zero or tiny scale: nvfp4_candidate on |x|, with the
// sign bits of the negative elements added.
__device__ __forceinline__ float nvfp4_candidate_tiny(const float* x, float a, float s_g, float c, uint64_t& codes) {
  float ax[16];
  uint64_t neg = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    ax[i] = fabsf(x[i]);
    neg |= static_cast<uint64_t>(x[i] < 0.0f) << (4 * i + 3);
  }
  uint64_t mags;
  uint32_t sf;
  const float err = nvfp4_candidate(ax, a, s_g, c, mags, sf);
  codes = mags | neg;
  return err;
}

// One candidate on the signed values x (the exact definition): rounding is
// symmetric in sign, so the magnitude codes, x - v S and its square are those
// of |x|, and the conversion supplies each element's sign bit (cleared by the
// caller where the magnitude is zero).  Zero and tiny scales take
// nvfp4_candidate on |x|.
__device__ __forceinline__ float nvfp4_candidate_s(const float* x, float a, float s_g, float c, float rden,
                                                   uint64_t& codes, uint32_t& sf) {
  sf = e4m3_code_of_quotient_r(a, __fmul_rn(c, s_g), rden);
  const float S = __fmul_rn(e4m3_decode(sf), s_g);
  if (!(S >= 0x1p-100f)) return nvfp4_candidate_tiny(x, a, s_g, c, codes);
  const float rS = __frcp_rn(S);
  float d2[16];
  uint32_t clo = 0, chi = 0;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    // both ends of both elements' brackets, two elements per conversion
    const float q0 = __fmul_rn(x[i], rS), q1 = __fmul_rn(x[i + 1], rS);
    const uint32_t lo = cvt_e2m1x2(__fmul_rn(q0, kBracketLo), __fmul_rn(q1, kBracketLo));
    const uint32_t hi = cvt_e2m1x2(__fmul_rn(q0, kBracketHi), __fmul_rn(q1, kBracketHi));
    uint32_t p = lo;
    if (lo != hi) {  // an end differs (never the sign): settle that element by the exact division
      const uint32_t m0 = ((lo ^ hi) & 0x7u) ? (e2m1_code_exact(fabsf(x[i]), S) | (lo & 0x8u)) : (lo & 0xFu);
      const uint32_t m1 =
          ((lo ^ hi) & 0x70u) ? ((e2m1_code_exact(fabsf(x[i + 1]), S) << 4) | (lo & 0x80u)) : (lo & 0xF0u);
      p = m0 | m1;
    }
    if (i < 8) clo |= p << (4 * i);
    else chi |= p << (4 * (i - 8));
    const float2 v = e2m1x2_decode(p);
    const float d0 = __fsub_rn(x[i], __fmul_rn(v.x, S));
    const float d1 = __fsub_rn(x[i + 1], __fmul_rn(v.y, S));
    d2[i] = __fmul_rn(d0, d0);
    d2[i + 1] = __fmul_rn(d1, d1);
  }
  codes = static_cast<uint64_t>(clo) | (static_cast<uint64_t>(chi) << 32);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int i = 0; i < w; ++i) d2[i] = __fadd_rn(d2[2 * i], d2[2 * i + 1]);
  }
  return d2[0];
}

// Signed codes -> block: the lower-error candidate (ties to 6), with the sign
// bit kept only where the magnitude code is non-zero (canonical +0).
__device__ __forceinline__ Nvfp4Block nvfp4_pick(float err6, uint64_t c6, uint32_t e6, float err4, uint64_t c4,
                                                 uint32_t e4) {
  const bool four = err4 < err6;
  const uint64_t codes = four ? c4 : c6;
  const uint64_t mags = codes & 0x7777777777777777ull;
  const uint64_t nz = (mags | (mags >> 1) | (mags >> 2)) & 0x1111111111111111ull;
  Nvfp4Block b;
  b.codes = mags | (codes & (nz << 3));
  b.sf = four ? e4 : e6;
  return b;
}

// NVFP4 4-vs-6 quantization of 16 float32 values with tensor scale s_g > 0.
__device__ __forceinline__ Nvfp4Block nvfp4_quantize16(const float* x, const Nvfp4Scale& ts) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  uint64_t c6, c4;
  uint32_t e6, e4;
  const float err6 = nvfp4_candidate_s(x, a, ts.s_g, 6.0f, ts.rd6, c6, e6);
  const float err4 = nvfp4_candidate_s(x, a, ts.s_g, 4.0f, ts.rd4, c4, e4);
  return nvfp4_pick(err6, c6, e6, err4, c4, e4);
}
__device__ __forceinline__ Nvfp4Block nvfp4_quantize16(const float* x, float s_g) {
  return nvfp4_quantize16(x, make_nvfp4_scale(s_g));
}

// The 4-vs-6 search for the requantization of h in the gate/up epilogue.
// Same block-scale codes (exact) as nvfp4_candidate; two departures from the
// definition, both for speed in the GEMM epilogue:
//   - the element quotient is RN(|x| * RN(1/S)) instead of RN(|x| / S),
//     converted two elements at a time.  The two differ by at most 2^-23
//     relative, so an element code can differ only where |x| / S lies that
//     close to a rounding midpoint of E2M1;
//   - the squared error is accumulated with fused multiply-adds, |x| - v S
//     and then its square added in, even and odd elements in two running
//     sums, instead of separately rounded products and a pairwise tree.
//     The sum differs from the definition's in its last bits, which can
//     change the pick only where the two candidates' errors nearly tie.
// The intermediate's parity bar (at most 1e-3 of its codes may differ, since
// h itself is computed in float32 with a fast exponential) absorbs both.
// Zero and tiny scales take the exact path.
//
// The signed values go through the conversion as they are: rounding is
// symmetric in sign, so the magnitude code, x - v S and its square are those
// of |x| and the conversion supplies the sign bit (cleared afterwards where
// the magnitude is zero).

// One candidate with a normal scale S: signed codes (element i in bits
// [4i, 4i+4)) and the squared error.
__device__ __forceinline__ float nvfp4_candidate_hs(const float* x, float S, uint64_t& codes) {
  const float rS = __frcp_rn(S);
  uint32_t clo = 0, chi = 0;
  float e0 = 0.0f, e1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const uint32_t p = cvt_e2m1x2(__fmul_rn(x[i], rS), __fmul_rn(x[i + 1], rS));
    if (i < 8) clo |= p << (4 * i);
    else chi |= p << (4 * (i - 8));
    const float2 v = e2m1x2_decode(p);
    const float d0 = __fmaf_rn(-v.x, S, x[i]);
    const float d1 = __fmaf_rn(-v.y, S, x[i + 1]);
    e0 = __fmaf_rn(d0, d0, e0);
    e1 = __fmaf_rn(d1, d1, e1);
  }
  codes = static_cast<uint64_t>(clo) | (static_cast<uint64_t>(chi) << 32);
  return __fadd_rn(e0, e1);
}

// NVFP4 4-vs-6 quantization of 16 values of h.
__device__ __forceinline__ Nvfp4Block nvfp4_quantize16_h(const float* x, const Nvfp4Scale& hs) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  const uint32_t e6 = e4m3_code_of_quotient_r(a, __fmul_rn(6.0f, hs.s_g), hs.rd6);
  const uint32_t e4 = e4m3_code_of_quotient_r(a, __fmul_rn(4.0f, hs.s_g), hs.rd4);
  const float S6 = __fmul_rn(e4m3_decode(e6), hs.s_g);
  const float S4 = __fmul_rn(e4m3_decode(e4), hs.s_g);
  uint64_t c6, c4;
  const float err6 = (S6 >= 0x1p-100f) ? nvfp4_candidate_hs(x, S6, c6) : nvfp4_candidate_tiny(x, a, hs.s_g, 6.0f, c6);
  const float err4 = (S4 >= 0x1p-100f) ? nvfp4_candidate_hs(x, S4, c4) : nvfp4_candidate_tiny(x, a, hs.s_g, 4.0f, c4);
  return nvfp4_pick(err6, c6, e6, err4, c4, e4);
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
    // two elements per conversion (same rounding and saturation as
    // e4m3_encode); a code whose magnitude bits are zero loses its sign bit
    const uint32_t p0 = cvt_e4m3x2(__fmul_rn(x[4 * w], scale), __fmul_rn(x[4 * w + 1], scale));
    const uint32_t p1 = cvt_e4m3x2(__fmul_rn(x[4 * w + 2], scale), __fmul_rn(x[4 * w + 3], scale));
    const uint32_t word = p0 | (p1 << 16);
    const uint32_t nonzero = ((word & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & 0x80808080u;
    words[w] = (word & 0x7F7F7F7Fu) | (word & nonzero);
  }
  return e;
}

}  // namespace moe
