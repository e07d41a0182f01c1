// Pieces of the persistent block-scaled GEMM kernel: tile constants, kernel
// arguments, the expert lookup and the epilogue that turns a 128-column slice
// of one accumulator row into outputs.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "quant.cuh"

namespace moe {

constexpr int kBM = 128;               // accumulator rows per CTA (one TMEM lane per row)
constexpr int kBN = 256;               // accumulator columns (weight rows of one tile)
constexpr int kRowBytesPerStage = 128;  // K bytes of one row per stage
constexpr int kEpiWarps = 8;             // two warps per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;

// B_ROWS: weight rows a CTA loads per stage.
template <int FMT, int B_ROWS, int STAGES>
struct GemmTraits {
  static constexpr bool kScaled = FMT != MOE_BF16;  // block-scaled formats carry scale atoms
  static constexpr int kStages = STAGES;
  static constexpr int kElemsPerStage = (FMT == MOE_NVFP4) ? 256 : (FMT == MOE_MXFP8 ? 128 : 64);
  static constexpr int kMmaK = (FMT == MOE_NVFP4) ? 64 : (FMT == MOE_MXFP8 ? 32 : 16);
  static constexpr int kSfVec = (FMT == MOE_NVFP4) ? 16 : 32;
  // scale bytes of 128 rows for one stage: NVFP4 16 scales/row = 4 atoms,
  // MXFP8 4 scales/row = 1 atom, BF16 none
  static constexpr int kSfBytes128 = kScaled ? 128 * (kElemsPerStage / kSfVec) : 0;
  static constexpr int kABytes = kBM * kRowBytesPerStage;
  static constexpr int kBBytes = B_ROWS * kRowBytesPerStage;
  static constexpr int kSfaOff = kABytes + kBBytes;
  static constexpr int kSfbOff = kSfaOff + kSfBytes128;
  // every CTA holds the scales of all kBN weight rows
  static constexpr int kStageRaw = kSfbOff + (kBN / 128) * kSfBytes128;
  static constexpr int kStageBytes = (kStageRaw + 1023) / 1024 * 1024;
  // TMEM columns: accumulator [0, kBN), scales of A, then scales of B
  static constexpr int kTmemSfa = kBN;
  static constexpr int kSfaCols = (FMT == MOE_NVFP4) ? 16 : 4;
  static constexpr int kTmemSfb = kTmemSfa + kSfaCols;
};

struct GemmArgs {
  const uint8_t* a_codes;     // tiled activation codes (128-row tiles)
  const uint8_t* b_codes;     // tiled weight codes (256-row tiles), expert 0
  const uint8_t* a_sf;
  const uint8_t* b_sf;
  const int32_t* offsets;
  const int32_t* counts;
  const float* a_scale;
  const float* w_scales;
  const float* h_scale;
  uint8_t* h_codes;
  uint8_t* h_sf;
  float* dbg;
  __nv_bfloat16* out;
  uint32_t* status;
  const int32_t* expert_map;  // optional: weights of row group e are expert_map[e]
  int n_weights;              // experts in the packed weights
  int E;                      // row groups (experts, or segments with an expert map)
  int K;            // reduction length in elements
  int n_rows_b;     // weight rows per expert (2I for gate/up, H for down)
  int64_t kb;                 // bytes of one code row, padded to a multiple of 128
  int64_t b_expert_stride;    // code bytes of one expert's weight matrix
  int64_t h_kb;               // gate/up: padded code-row bytes of h
  int64_t sf_rb_stride;       // scale bytes of one 128-row block (= K / sfvec * 128)
  int64_t b_sf_expert_stride; // scale bytes of one expert's weight matrix
};

__device__ __forceinline__ int find_expert(const int32_t* offs, int E, int row) {
  int lo = 0, hi = E;  // offs[lo] <= row < offs[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offs[mid] <= row) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Two 16-byte chunks c0, c1 of a row at logical bytes [byte, byte + 32) of the
// tiled layout (byte a multiple of 32) in one 32-byte store: the 128-byte
// swizzle keeps the pair in one aligned 32-byte slot, in order when the row's
// swizzle key (row % 8) is even and swapped when it is odd.  base must be
// 32-byte aligned.
__device__ __forceinline__ void store_tiled32(uint8_t* base, int64_t row, int64_t byte, int64_t kb, int64_t TR,
                                              uint4 c0, uint4 c1) {
  const int64_t o0 = tile_offset(row, byte, kb, TR);
  const bool swap = ((row % TR) & 1) != 0;
  const uint4 lo = swap ? c1 : c0, hi = swap ? c0 : c1;
  const uint32_t v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  st_global_v8(base + (swap ? o0 - 16 : o0), v);
}

// Epilogue of one accumulator row slice: acc holds columns
// [half * kBN/2, (half + 1) * kBN/2) of row `row` (weight tile nt, expert e).
//   gate/up: tensor scales, SwiGLU, requantization of h (NVFP4 4-vs-6 or
//            MXFP8), optional float32 copy of g and u;
//   down:    tensor scales, bf16 store.
template <int FMT, bool GATEUP>
__device__ __forceinline__ void epilogue_rows(const GemmArgs& args, float* acc, int64_t row, int e, int nt,
                                              int half) {
  const int I = args.n_rows_b / 2;  // gate/up: channels
  const int H = args.n_rows_b;      // down: output channels
  if (GATEUP && FMT == MOE_BF16) {
    // columns of this half: [gate 32 | up 32] x 2, channels ch0 + [0, 64);
    // h in bf16 fills one 128-byte row of h's K tile ch0 / 64
    const int ch0 = nt * (kBN / 2) + half * (kBN / 4);
    uint32_t p[32];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float* g = acc + 64 * j;
      float* u = acc + 64 * j + 32;
      if (args.dbg != nullptr) {
        float4* dg = reinterpret_cast<float4*>(args.dbg + row * (2 * I) + ch0 + 32 * j);
        float4* du = reinterpret_cast<float4*>(args.dbg + row * (2 * I) + I + ch0 + 32 * j);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dg[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
          du[i] = make_float4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float h0 = __fdividef(g[2 * i] * u[2 * i], 1.0f + __expf(-g[2 * i]));
        const float h1 = __fdividef(g[2 * i + 1] * u[2 * i + 1], 1.0f + __expf(-g[2 * i + 1]));
        const __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
        p[16 * j + i] = *reinterpret_cast<const uint32_t*>(&b);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(args.h_codes + tile_offset(row, 2 * ch0 + 16 * c, args.h_kb, kActTileRows)) =
          make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
  } else if (GATEUP) {
    // columns of this half: [gate 32 | up 32] x 2, channels ch0 + [0, 64)
    const int ch0 = nt * (kBN / 2) + half * (kBN / 4);
    const float sa = (FMT == MOE_NVFP4) ? __ldg(args.a_scale) : 1.0f;
    const float sg = (FMT == MOE_NVFP4) ? __fmul_rn(sa, __ldg(args.w_scales + 3 * e + 0)) : 1.0f;
    const float su = (FMT == MOE_NVFP4) ? __fmul_rn(sa, __ldg(args.w_scales + 3 * e + 1)) : 1.0f;
    const float sh = (FMT == MOE_NVFP4) ? __ldg(args.h_scale) : 1.0f;
    const Nvfp4Scale hs = make_nvfp4_scale(sh);
#pragma unroll
    for (int j = 0; j < kBN / 128; ++j) {
      float* g = acc + 64 * j;
      float* u = acc + 64 * j + 32;
      const int ch = ch0 + 32 * j;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        g[i] *= sg;
        u[i] *= su;
      }
      if (args.dbg != nullptr) {
        float4* dg = reinterpret_cast<float4*>(args.dbg + row * (2 * I) + ch);
        float4* du = reinterpret_cast<float4*>(args.dbg + row * (2 * I) + I + ch);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dg[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
          du[i] = make_float4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
        }
      }
      // h = silu(g) * u, written over g
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = __fdividef(g[i] * u[i], 1.0f + __expf(-g[i]));
    }
    // h of this thread: acc[0..32) channels ch0 + [0, 32), acc[64..96) ch0 + [32, 64)
    // the thread's 64 channels: NVFP4 4 blocks = 32 code bytes + 4 adjacent
    // scale bytes, MXFP8 2 blocks = 2 x 32 code bytes + 2 adjacent scale bytes
    const bool wide = (reinterpret_cast<uintptr_t>(args.h_codes) & 31u) == 0u;
    if (FMT == MOE_NVFP4) {
      uint32_t cw[8];
      uint32_t sfw = 0;
#pragma unroll 1
      for (int b2 = 0; b2 < 2; ++b2) {
        float blk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[i] = (b2 == 0) ? acc[i] : acc[64 + i];
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          const int b = 2 * b2 + jb;
          const Nvfp4Block qb = nvfp4_quantize16_h(blk + 16 * jb, hs);
          const uint32_t lo = static_cast<uint32_t>(qb.codes), hi = static_cast<uint32_t>(qb.codes >> 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j == b) {
              cw[2 * j] = lo;
              cw[2 * j + 1] = hi;
            }
          }
          sfw |= (qb.sf & 0xFFu) << (8 * b);
          if (!wide) {
            const int ch = ch0 + 16 * b;
            *reinterpret_cast<uint2*>(args.h_codes + tile_offset(row, ch / 2, args.h_kb, kActTileRows)) =
                make_uint2(lo, hi);
          }
        }
      }
      if (wide)
        store_tiled32(args.h_codes, row, ch0 / 2, args.h_kb, kActTileRows, make_uint4(cw[0], cw[1], cw[2], cw[3]),
                      make_uint4(cw[4], cw[5], cw[6], cw[7]));
      // blocks ch0 / 16 .. + 3: four adjacent bytes of one scale atom row
      *reinterpret_cast<uint32_t*>(args.h_sf + sf_offset(row, ch0 / 16, I / 16)) = sfw;
    } else {
      uint32_t sfw = 0;
#pragma unroll 1
      for (int b = 0; b < 2; ++b) {
        float blk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[i] = (b == 0) ? acc[i] : acc[64 + i];
        uint32_t w[8];
        const uint32_t ex = mxfp8_quantize32(blk, w);
        const int ch = ch0 + 32 * b;
        if (wide) {
          store_tiled32(args.h_codes, row, ch, args.h_kb, kActTileRows, make_uint4(w[0], w[1], w[2], w[3]),
                        make_uint4(w[4], w[5], w[6], w[7]));
        } else {
          *reinterpret_cast<uint4*>(args.h_codes + tile_offset(row, ch, args.h_kb, kActTileRows)) =
              make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(args.h_codes + tile_offset(row, ch + 16, args.h_kb, kActTileRows)) =
              make_uint4(w[4], w[5], w[6], w[7]);
        }
        sfw |= (ex & 0xFFu) << (8 * b);
      }
      // blocks ch0 / 32, + 1: two adjacent bytes of one scale atom row
      *reinterpret_cast<uint16_t*>(args.h_sf + sf_offset(row, ch0 / 32, I / 32)) = static_cast<uint16_t>(sfw);
    }
  } else {
    const float s = (FMT == MOE_NVFP4) ? __fmul_rn(__ldg(args.a_scale), __ldg(args.w_scales + 3 * e + 2)) : 1.0f;
    (void)I;
    __nv_bfloat16* dst = args.out + row * H + nt * kBN + half * (kBN / 2);
    if ((reinterpret_cast<uintptr_t>(args.out) & 31u) == 0u) {
      // the row's 256 bytes as eight whole 32-byte sectors
#pragma unroll
      for (int i = 0; i < kBN / 32; ++i) {
        uint32_t p[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(acc[16 * i + 2 * c] * s, acc[16 * i + 2 * c + 1] * s);
          p[c] = *reinterpret_cast<const uint32_t*>(&b);
        }
        st_global_v8(dst + 16 * i, p);
      }
    } else {
#pragma unroll
      for (int i = 0; i < kBN / 16; ++i) {
        uint32_t p[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(acc[8 * i + 2 * c] * s, acc[8 * i + 2 * c + 1] * s);
          p[c] = *reinterpret_cast<const uint32_t*>(&b);
        }
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(p[0], p[1], p[2], p[3]);
      }
    }
  }
}

}  // namespace moe
