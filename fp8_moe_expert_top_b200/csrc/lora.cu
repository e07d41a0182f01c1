// LoRA "shrink" of the BF16 experts: z = s_e * (a A_e^T) for every
// 128-row block of permuted rows (a = the rows of x, or of the intermediate
// h), written as bf16 into the extra 64-element K tile that every row of
// these operands carries.  The following GEMM then runs over K + 64: its
// weight rows hold B_e in that tile, so the adapter's "expand" B_e z is summed
// by the same MMAs as the main product, W_e a + s_e B_e (A_e a).
//
// Pages: "thinkingmachines/Inkling-2-Small", section Configurations, and
// "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
// section "LoRA and reinforcement learning": adapters on the routed experts
// need BF16 expert weights; the pages' validation run used rank 32.  An
// adapter here has rank <= 32: the A rows of gate (0-31) and up (32-63) share
// one N = 64 product; the down adapter uses rows 0-31 (rows 32-63 are zero).
//
// One CTA per 128-row block (blocks past the rows in use exit at once):
//   warp 0     producer: 1-D bulk copies of the row block's tile of a (rows in
//              use, rounded up to 16) and of the expert's 64 A rows, per
//              64-element K step, into a 4-stage ring
//   warp 1     MMA: tcgen05.mma kind::f16, M = 128, N = 64, fp32 in TMEM
//   warps 2-5  epilogue: tcgen05.ld of the 64 columns of one row, times s_e,
//              bf16, one 128-byte row of the adapter K tile
// Every wait is bounded (status bits on expiry), work in flight is drained
// before TMEM is freed.
#include <cstdint>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kLStages = 4;
constexpr int kLN = 64;                       // adapter rows (gate + up, or down + zeros)
constexpr int kLThreads = 64 + 32 * 4;
constexpr int kLABytes = 128 * 128;           // a: 128 rows x 128 bytes
constexpr int kLBBytes = kLN * 128;           // A: 64 rows x 128 bytes
constexpr int kLStageBytes = kLABytes + kLBBytes;

struct ShrinkArgs {
  uint8_t* a;               // tiled bf16 rows, kb bytes per row (K + 64 elements)
  const uint8_t* w;         // [E][64 x 2K] A rows of each expert, tiled 64 rows
  const float* scales;      // [E][3]: adapter scaling in [e][0]
  const int32_t* offsets;   // [E + 1]
  const int32_t* counts;    // [E]
  const int32_t* expert_map;  // optional [E]: row group -> expert of the weights
  int n_weights;
  uint32_t* status;
  int E, K;
  int64_t kb;               // bytes of one row of a (2K + 128)
};

__global__ void __launch_bounds__(kLThreads, 1) lora_shrink_kernel(const ShrinkArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kLStages * kLStageBytes);
  uint64_t* empty_bar = full_bar + kLStages;
  uint64_t* acc_bar = empty_bar + kLStages;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* s_info = reinterpret_cast<int*>(tmem_slot + 4);   // expert, rows in use

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    const int rows_total = args.offsets[args.E];
    int e = -1, valid = 0;
    if (rb * 128 < rows_total) {
      e = find_expert(args.offsets, args.E, rb * 128);
      valid = min(128, args.offsets[e] + args.counts[e] - rb * 128);
    }
    s_info[0] = e;
    s_info[1] = valid;
  }
  __syncthreads();
  const int e = s_info[0], valid = s_info[1];
  if (e < 0 || valid <= 0) return;    // a block past the rows in use, or a padding-only block
  int we = e;                         // expert whose adapter applies
  if (args.expert_map != nullptr) {
    we = __ldg(args.expert_map + e);
    if (we < 0 || we >= args.n_weights) {
      if (threadIdx.x == 0 && args.status != nullptr) atomicOr(args.status, MOE_DEVICE_BAD_GROUP_EXPERT);
      we = 0;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kLN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int k_tiles = args.K / 64;
  const int64_t ktiles_row = args.kb >> 7;
  uint32_t fail_bits = 0, armed = 0u, armed_par = 0u;

  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* a_tiles = args.a + static_cast<int64_t>(rb) * ktiles_row * kLABytes;
      const uint8_t* w_tiles = args.w + static_cast<int64_t>(we) * k_tiles * kLBBytes;
      const uint32_t a_bytes = static_cast<uint32_t>((valid + 15) / 16) * 16 * 128;
      const uint64_t pol = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
          break;
        }
        uint8_t* st = smem + stage * kLStageBytes;
        mbar_arrive_expect_tx(&full_bar[stage], a_bytes + kLBBytes);
        bulk_load(st, a_tiles + static_cast<int64_t>(kt) * kLABytes, a_bytes, &full_bar[stage], pol);
        bulk_load(st + kLABytes, w_tiles + static_cast<int64_t>(kt) * kLBBytes, kLBBytes, &full_bar[stage], pol);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kLStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kLN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + stage * kLStageBytes);
        const uint64_t adesc = make_desc_sw128(st), bdesc = make_desc_sw128(st + kLABytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem_base, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kt | kk) != 0 ? 1u : 0u);
        tc_commit(&empty_bar[stage]);
        if (++stage == kLStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit(acc_bar);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    if (mbar_wait(acc_bar, 0, abort_flag)) {
      tc_fence_after();
      float z[64];
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      tmem_ld32(t_row, z);
      tmem_ld32(t_row + 32, z + 32);
      tmem_ld_wait();
      if (row < valid) {
        const float s = __ldg(args.scales + 3 * we);
        uint32_t p[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(z[2 * i] * s, z[2 * i + 1] * s);
          p[i] = *reinterpret_cast<const uint32_t*>(&b);
        }
        const int64_t r = static_cast<int64_t>(rb) * 128 + row;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(args.a + tile_offset(r, 2 * static_cast<int64_t>(args.K) + 16 * c, args.kb,
                                                         kActTileRows)) =
              make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
      }
    } else {
      fail_bits |= MOE_DEVICE_TIMEOUT_EPILOGUE;
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    bool drained = true;
    if (warp == 0 && lane == 0) {
      for (int st = 0; st < kLStages; ++st)
        if ((armed >> st) & 1u) drained = mbar_wait_drain(&full_bar[st], (armed_par >> st) & 1u) && drained;
    } else if (warp == 1 && lane == 0) {
      tc_commit(drain_bar);
      drained = mbar_wait_drain(drain_bar, 0);
    }
    if (!drained) *drain_failed = 1;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (warp == 1 && !*drain_failed) {
    __syncwarp();
    tmem_dealloc(tmem_base, kLN);
  }
}

}  // namespace

cudaError_t launch_lora_shrink(uint8_t* a, int64_t kb, int K, const uint8_t* w, const float* scales,
                               const int32_t* offsets, const int32_t* counts, const int32_t* expert_map,
                               int n_weights, int E, int64_t R_max, uint32_t* status, cudaStream_t stream) {
  if (R_max <= 0) return cudaSuccess;
  constexpr size_t smem = 1024 + kLStages * kLStageBytes + (2 * kLStages + 2) * 8 + 32;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(lora_shrink_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return attr_err;
  ShrinkArgs args;
  args.a = a;
  args.w = w;
  args.scales = scales;
  args.offsets = offsets;
  args.counts = counts;
  args.expert_map = expert_map;
  args.n_weights = n_weights;
  args.status = status;
  args.E = E;
  args.K = K;
  args.kb = kb;
  return launch_pdl(lora_shrink_kernel, dim3(static_cast<unsigned>(R_max / 128)), dim3(kLThreads), smem, stream,
                    args);
}

}  // namespace moe
