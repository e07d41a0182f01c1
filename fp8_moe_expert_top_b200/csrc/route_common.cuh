// Routing pieces shared by the top-k kernel over given logits and the fused
// router (GEMM + top-k): the softmax's exponential.
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

}  // namespace moe
