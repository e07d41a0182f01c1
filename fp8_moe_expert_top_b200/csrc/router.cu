// Router scores fused with the top-k: logits = x W_r^T on tcgen05, and in
// the same kernel the per-token top-k, the softmax over the k selected scores
// and the per-expert token bitmaps that the slot sort counts.
//
// Pages: "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview,
// and "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
// section "NVFP4 and MXFP8 experts": every token is scored against the 384
// routed experts and sent to the 8 best.  The scores never reach global
// memory (unless the caller asks for a debug copy): the accumulator in TMEM
// is reduced to the k selected experts by the epilogue.
//
// Large batches (router_topk_kernel), one CTA per 128 tokens:
//   warp 0      producer: TMA tile loads (cp.async.bulk.tensor, 128-byte
//               swizzle, no multicast) of 64 bf16 of K for the 128 token rows
//               of x and for all expert rows of W_r, into a ring of stages
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//               M = 128, N = 256 and/or 128 per 128-expert block, the
//               accumulator of all (up to 512) experts in TMEM
//   warps 2-9   epilogue: two warps per TMEM lane quarter, one token row per
//               thread, half of its scores each: tcgen05.ld 32 scores at a
//               time, the top 8 kept in registers as order-preserving keys
//               (strictly-above insertion while scanning experts in
//               ascending order, so equal scores keep the lower index); the
//               halves merged through shared memory; then the same softmax
//               and bitmap update as route_topk_kernel (bit-identical
//               weights for equal scores).
// Mid-size batches (router_pair_kernel): the same with the experts split
// over a cluster of two CTAs per 128 tokens, the two top-8 lists merged
// through distributed shared memory.  Small batches (router_split_kernel):
// K split over a cluster of 4 or 8 CTAs per 128 tokens.
// Every wait is bounded; a wait that runs out raises the CTA's abort flag,
// the roles stop, work in flight is drained and a status bit is set.
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "pair.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

constexpr int kRM = 128;           // tokens per CTA (TMEM lanes)
constexpr int kRKElems = 64;       // bf16 of K per stage (128 bytes per row)
// Epilogue warps: two per TMEM lane quarter, each taking half of a row's
// score columns (one warp per quarter scanning all of them took as long as
// the MMAs at prefill, and pushed the partial scores half as fast at decode).
constexpr int kREpiWarps = 8;
constexpr int kRThreads = 64 + 32 * kREpiWarps;
constexpr int kRTileBytes = kRM * 128;  // one 128-row x 128-byte tile

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* tmap, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

struct RouterArgs {
  float* logits_out;  // optional [T][E] debug copy of the scores
  int32_t* topk_ids;
  float* topk_w;
  uint32_t* bitmap;   // [E][W] token bitmaps
  uint32_t* status;
  int T, E, H, k, W;
};

// Orders this thread's later generic-proxy accesses to shared memory after
// earlier async-proxy (bulk copy) writes to the same region.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Insert (key, e) into a row's top 8 (keys largest first), key strictly above
// tk[7]: all eight slots are updated at once from the old list (independent
// comparisons, not a chain of swaps); an equal key already held stays ahead.
__device__ __forceinline__ void topk_insert(uint32_t* tk, int* ti, uint32_t key, int e) {
  bool above[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) above[j] = key > tk[j];
#pragma unroll
  for (int j = 7; j > 0; --j) {
    tk[j] = above[j - 1] ? tk[j - 1] : (above[j] ? key : tk[j]);
    ti[j] = above[j - 1] ? ti[j - 1] : (above[j] ? e : ti[j]);
  }
  tk[0] = above[0] ? key : tk[0];
  ti[0] = above[0] ? e : ti[0];
}

// Row t's outputs from its top 8 (keys largest first): the softmax over the
// k selected scores as route_topk_kernel computes it (e_j = exp(l_j - l_0),
// summed in rank order, one division each), the ids, and the token's bit in
// each selected expert's bitmap (when the bitmaps are kept).
__device__ __forceinline__ void write_row_topk(const RouterArgs& args, int t, const uint32_t* tk, const int* ti) {
  const int k = args.k;
  float ex[8];
  float s = 0.0f;
  const float top = key_logit(tk[0]);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ex[j] = (j < k) ? exp_own(__fsub_rn(key_logit(tk[j]), top)) : 0.0f;
    if (j == 0) s = ex[0];
    else if (j < k) s = __fadd_rn(s, ex[j]);
  }
  const int64_t o = static_cast<int64_t>(t) * k;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      args.topk_ids[o + j] = ti[j];
      args.topk_w[o + j] = __fdiv_rn(ex[j], s);
      if (args.bitmap != nullptr)
        atomicOr(&args.bitmap[static_cast<int64_t>(ti[j]) * args.W + (t >> 5)], 1u << (t & 31));
    }
  }
}

// NB: 128-expert blocks of W_r (1..4); ST: ring stages.
template <int NB, int ST>
__global__ void __launch_bounds__(kRThreads, 1)
    router_topk_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       const RouterArgs args) {
  constexpr int kStageBytes = kRTileBytes * (1 + NB);
  constexpr uint32_t kTmemCols = NB == 1 ? 128u : (NB == 2 ? 256u : 512u);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + ST * kStageBytes);
  uint64_t* empty_bar = full_bar + ST;
  uint64_t* acc_bar = empty_bar + ST;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRM;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int k_tiles = args.H / kRKElems;
  uint32_t fail_bits = 0;
  uint32_t armed = 0u, armed_par = 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
          break;
        }
        uint8_t* st = smem + stage * kStageBytes;
        // a box that reaches past the last token or expert is filled with
        // zeros and still counts its full size
        mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
        tma_load_2d(st, &tmap_x, kt * kRKElems, m0, &full_bar[stage]);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          tma_load_2d(st + kRTileBytes * (1 + b), &tmap_w, kt * kRKElems, b * 128, &full_bar[stage]);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint64_t adesc0 = make_desc_sw128(smem_u32(smem));
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          ok = false;
          break;
        }
        tc_fence_after();
        // stage descriptors from stage 0's by a constant offset, MMAs unrolled
        const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage) * (kStageBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kRKElems / 16; ++kk) {
          const uint32_t acc = (kt | kk) != 0 ? 1u : 0u;
#pragma unroll
          for (int b = 0; b < NB; b += 2) {
            const uint64_t bdesc = adesc + (static_cast<uint64_t>(kRTileBytes * (1 + b)) >> 4);
            if (b + 1 < NB)
              tc_mma_bf16(tmem_base + 128 * b, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16(256), acc);
            else
              tc_mma_bf16(tmem_base + 128 * b, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16(128), acc);
          }
        }
        tc_commit(&empty_bar[stage]);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit(acc_bar);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warps 2..9: quarter q = warp % 4 of the TMEM lanes (rows), half of the
    // score columns (experts [half E/2, ...)).  Each keeps its row's top 8 of
    // its half; the second half's lists go through shared memory (the ring
    // is idle once the accumulator is complete) to the first half's warp,
    // which merges them, then computes the softmax and writes the row.
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int t = m0 + row;
    const bool acc_ok = mbar_wait(acc_bar, 0, abort_flag);
    if (!acc_ok) fail_bits |= MOE_DEVICE_TIMEOUT_EPILOGUE;
    // this row's top 8 so far as order-preserving keys, largest first; an
    // empty slot holds key 0, below every score
    uint32_t tk[8];
    int ti[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      tk[j] = 0u;
      ti[j] = 0;
    }
    if (acc_ok) {
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const int c0 = half * (NB * 2);
#pragma unroll 1
      for (int c = c0; c < c0 + NB * 2; ++c) {
        float v[32];
        tmem_ld32(t_row + 32 * c, v);
        tmem_ld_wait();
        if (t < args.T) {
          if (args.logits_out != nullptr) {
            float* dst = args.logits_out + static_cast<int64_t>(t) * args.E;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * c + i < args.E) dst[32 * c + i] = v[i];
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = 32 * c + i;
            const uint32_t key = e < args.E ? logit_key(v[i]) : 0u;
            // experts arrive in ascending order, so an equal score already
            // held keeps its lower index ahead
            if (key > tk[7]) topk_insert(tk, ti, key, e);
          }
        }
      }
    }
    uint32_t* xk = reinterpret_cast<uint32_t*>(smem);  // [128 rows][8] keys of the second half
    int* xi = reinterpret_cast<int*>(smem + kRM * 8 * 4);
    if (half == 1) {
      fence_proxy_async_shared();  // the ring last held bulk-copied operands
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        xk[row * 8 + j] = tk[j];
        xi[row * 8 + j] = ti[j];
      }
    }
    // both warps of the quarter arrive here exactly once, whatever happened
    asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(64) : "memory");
    if (half == 0 && acc_ok) {
      // merge: the second half's experts all have higher indices, so an
      // equal score goes after the first half's (strictly-above insertion)
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t key = xk[row * 8 + jj];
        const int e = xi[row * 8 + jj];
        if (key > tk[7] && e >= 0 && e < args.E) topk_insert(tk, ti, key, e);
      }
      if (t < args.T) {
        write_row_topk(args, t, tk, ti);
      }
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    // drain what is in flight before TMEM is freed (as in the expert GEMMs)
    bool drained = true;
    if (warp == 0 && lane == 0) {
      for (int st = 0; st < ST; ++st)
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
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Small batches: the same scores with K split over a cluster of KS CTAs per
// 128 tokens, so that a decode batch spreads its router weights over KS SMs
// instead of one.  CTA r of the cluster accumulates k tiles
// [r KT/KS, (r+1) KT/KS) of all NB expert blocks in TMEM.  After every CTA's
// MMAs are complete (first cluster barrier) each valid token row's partial
// scores are pushed (st.shared::cluster) into the ring of the CTA that owns
// the row, slot r of it; the tile's t_tile valid rows are shared out evenly
// (owner r holds rows [r rpo, (r+1) rpo), rpo = ceil(t_tile / KS) <= 128 /
// KS).  After the second cluster barrier each owner sums the KS partials of
// its rows in rank order (so the scores do not depend on timing) and a warp
// per row selects the top-k with warp_topk_keys (the largest scores, ties to
// the lower index).  The softmax and the bitmap update are those of
// route_topk_kernel.  Every thread passes both cluster barriers exactly once,
// whatever happened before, so a CTA that timed out cannot stall the others.
template <int NB, int ST, int KS>
__global__ void __launch_bounds__(kRThreads, 1)
    router_split_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                        const RouterArgs args) {
  constexpr int kStageBytes = kRTileBytes * (1 + NB);
  constexpr uint32_t kTmemCols = NB == 1 ? 128u : (NB == 2 ? 256u : 512u);
  constexpr int EP = NB * 128;     // scores per row in the receive slots
  constexpr int RPO = kRM / KS;    // rows owned by each CTA
  static_assert(KS * RPO * EP * 4 <= ST * kStageBytes, "receive slots must fit in the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* recv = reinterpret_cast<float*>(smem);  // [KS][RPO][EP], 16-byte units XOR-swizzled by row
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + ST * kStageBytes);
  uint64_t* empty_bar = full_bar + ST;
  uint64_t* acc_bar = empty_bar + ST;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int m0 = static_cast<int>(blockIdx.x / KS) * kRM;
  const int kt_per = (args.H / kRKElems) / KS;
  const int kt0 = static_cast<int>(rank) * kt_per;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint32_t fail_bits = 0;
  uint32_t armed = 0u, armed_par = 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = kt0; kt < kt0 + kt_per; ++kt) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
          break;
        }
        uint8_t* st = smem + stage * kStageBytes;
        mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
        tma_load_2d(st, &tmap_x, kt * kRKElems, m0, &full_bar[stage]);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          tma_load_2d(st + kRTileBytes * (1 + b), &tmap_w, kt * kRKElems, b * 128, &full_bar[stage]);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < kt_per; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + stage * kStageBytes);
        const uint64_t adesc = make_desc_sw128(st);
#pragma unroll
        for (int kk = 0; kk < kRKElems / 16; ++kk) {
          const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
#pragma unroll
          for (int b = 0; b < NB; b += 2) {
            const uint64_t bdesc = make_desc_sw128(st + kRTileBytes * (1 + b));
            if (b + 1 < NB)
              tc_mma_bf16(tmem_base + 128 * b, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16(256), acc);
            else
              tc_mma_bf16(tmem_base + 128 * b, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16(128), acc);
          }
        }
        tc_commit(&empty_bar[stage]);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit(acc_bar);
    }
  } else {
    // ------------------------------------------------------------ epilogue: accumulator complete
    if (!mbar_wait(acc_bar, 0, abort_flag)) fail_bits |= MOE_DEVICE_TIMEOUT_EPILOGUE;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    // drain what is in flight before the ring is overwritten and TMEM freed
    bool drained = true;
    if (warp == 0 && lane == 0) {
      for (int st = 0; st < ST; ++st)
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
  const bool acc_ok = !*abort_flag;
  cluster_sync();  // every CTA's MMAs are complete: all rings may be written

  // The tile's valid rows are shared out evenly: owner r holds rows
  // [r rpo, (r + 1) rpo) of the t_tile valid ones (rpo <= RPO), so a batch
  // smaller than 128 tokens spreads its rows, and its top-k work, over all
  // KS CTAs, and rows past the batch are neither pushed nor reduced.
  const int t_tile = min(kRM, args.T - m0);
  const int rpo = (t_tile + KS - 1) / KS;
  if (warp >= 2 && acc_ok && (warp & 3) * 32 < t_tile) {
    // push this CTA's partial scores of each row into the row's owner; two
    // warps per TMEM lane quarter, half of the score columns each
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    // rows past the batch push nothing; their owner is set to this CTA only
    // so that the address below is computed for a rank of the cluster
    const uint32_t owner = row < t_tile ? static_cast<uint32_t>(row / rpo) : rank;
    const int r_loc = row < t_tile ? row % rpo : 0;
    const uint32_t dst = mapa_shared(smem_u32(recv), owner) +
                         static_cast<uint32_t>(((static_cast<int>(rank) * RPO + r_loc) * EP) * 4);
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
    for (int c = half * (NB * 2); c < (half + 1) * (NB * 2); ++c) {
      float v[32];
      tmem_ld32(t_row + 32 * c, v);
      tmem_ld_wait();
      if (row < t_tile) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t unit = static_cast<uint32_t>(8 * c + u) ^ static_cast<uint32_t>(r_loc & 7);
          st_cluster_v4(dst + 16u * unit, v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // every partial has arrived at its owner
  tc_fence_after();

  {
    // reduce the owned rows over the KS partials, then top-k (a warp per row,
    // every warp of the CTA)
    const int own0 = static_cast<int>(rank) * rpo;
    for (int r_loc = warp; r_loc < rpo && own0 + r_loc < t_tile; r_loc += kRThreads / 32) {
      const int t = m0 + own0 + r_loc;
      uint32_t key[EP / 32];
#pragma unroll
      for (int i = 0; i < EP / 32; ++i) {
        const int e = 32 * i + lane;
        const int off = 4 * ((e >> 2) ^ (r_loc & 7)) + (e & 3);
        float v = recv[(0 * RPO + r_loc) * EP + off];
#pragma unroll
        for (int s = 1; s < KS; ++s) v = __fadd_rn(v, recv[(s * RPO + r_loc) * EP + off]);
        key[i] = 0u;
        if (e < args.E) {
          if (args.logits_out != nullptr) args.logits_out[static_cast<int64_t>(t) * args.E + e] = v;
          key[i] = logit_key(v);
        }
      }
      // top-k and softmax as route_topk_kernel computes them
      const int k = args.k;
      int si[8];
      const uint32_t my_key = warp_topk_keys<EP / 32>(key, k, lane, si);
      const float w = warp_topk_softmax(key_logit(my_key), k, lane);
      const int64_t o = static_cast<int64_t>(t) * k;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && lane == j) {
          args.topk_ids[o + j] = si[j];
          args.topk_w[o + j] = w;
          if (args.bitmap != nullptr)
            atomicOr(&args.bitmap[static_cast<int64_t>(si[j]) * args.W + (t >> 5)], 1u << (t & 31));
        }
      }
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  if (warp == 1 && !*drain_failed) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Mid-size batches (too many row tiles for the K split, fewer than one per
// pair of SMs): the experts split over a cluster of two CTAs per 128 tokens.
// CTA r computes the scores of experts [r NH, (r+1) NH) over all of K (N = NH
// per MMA, NH = E/2), so each CTA streams half of W_r and no partial scores
// move.  Its epilogue (two warps per TMEM lane quarter, half of its columns
// each) keeps each row's top 8 as keys and merges the two halves through its
// idle ring; after a first cluster barrier CTA 1 sends its lists
// (st.shared::cluster, 64 bytes per row) into CTA 0's ring, and after a
// second one CTA 0 merges them (its experts come first, so an equal score
// keeps the lower index), computes the softmax and writes the row.  Every
// thread passes both cluster barriers exactly once, whatever happened before.
template <int NC, int ST>
__global__ void __launch_bounds__(kRThreads, 1)
    router_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       const RouterArgs args) {
  constexpr int NH = 32 * NC;                  // experts (MMA N) per CTA
  constexpr int kWBytes = NH * 128;            // one stage of this CTA's W_r rows
  constexpr int kStageBytes = kRTileBytes + kWBytes;
  constexpr uint32_t kTmemCols = NH <= 32 ? 32u : (NH <= 64 ? 64u : (NH <= 128 ? 128u : 256u));
  static_assert(NC % 2 == 0 && NH <= 256, "two selecting warps per quarter, N <= 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + ST * kStageBytes);
  uint64_t* empty_bar = full_bar + ST;
  uint64_t* acc_bar = empty_bar + ST;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);
  // exchange areas in the ring: xk, xi once this CTA's MMAs are complete;
  // rk, ri once both CTAs' are (after the first cluster barrier)
  uint32_t* xk = reinterpret_cast<uint32_t*>(smem);             // [128][8] keys, second half of this CTA
  int* xi = reinterpret_cast<int*>(smem + kRM * 8 * 4);         // [128][8] experts
  uint32_t* rk = reinterpret_cast<uint32_t*>(smem + kRM * 64);  // [128][8] keys from CTA 1 (CTA 0 only)
  int* ri = reinterpret_cast<int*>(smem + kRM * 96);            // [128][8] experts from CTA 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int m0 = static_cast<int>(blockIdx.x >> 1) * kRM;
  const int e0 = static_cast<int>(rank) * NH;  // this CTA's first expert
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int k_tiles = args.H / kRKElems;
  uint32_t fail_bits = 0;
  uint32_t armed = 0u, armed_par = 0u;
  uint32_t tk[8];
  int ti[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    tk[j] = 0u;
    ti[j] = 0;
  }
  bool acc_ok = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
          break;
        }
        uint8_t* st = smem + stage * kStageBytes;
        mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
        tma_load_2d(st, &tmap_x, kt * kRKElems, m0, &full_bar[stage]);
        tma_load_2d(st + kRTileBytes, &tmap_w, kt * kRKElems, e0, &full_bar[stage]);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint64_t adesc0 = make_desc_sw128(smem_u32(smem));
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage) * (kStageBytes >> 4);
        const uint64_t bdesc = adesc + (kRTileBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kRKElems / 16; ++kk)
          tc_mma_bf16(tmem_base, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16(NH), (kt | kk) != 0 ? 1u : 0u);
        tc_commit(&empty_bar[stage]);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit(acc_bar);
    }
  } else {
    // ------------------------------------------------------------ epilogue: this CTA's top 8 per row
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int t = m0 + row;
    acc_ok = mbar_wait(acc_bar, 0, abort_flag);
    if (!acc_ok) fail_bits |= MOE_DEVICE_TIMEOUT_EPILOGUE;
    if (acc_ok) {
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = half * (NC / 2); c < (half + 1) * (NC / 2); ++c) {
        float v[32];
        tmem_ld32(t_row + 32 * c, v);
        tmem_ld_wait();
        if (t < args.T) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = e0 + 32 * c + i;
            if (args.logits_out != nullptr && e < args.E) args.logits_out[static_cast<int64_t>(t) * args.E + e] = v[i];
            const uint32_t key = e < args.E ? logit_key(v[i]) : 0u;
            if (key > tk[7]) topk_insert(tk, ti, key, e);
          }
        }
      }
    }
    if (half == 1) {
      fence_proxy_async_shared();  // the ring last held bulk-copied operands
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        xk[row * 8 + j] = tk[j];
        xi[row * 8 + j] = ti[j];
      }
    }
    // both warps of the quarter arrive here exactly once, whatever happened
    asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(64) : "memory");
    if (half == 0 && acc_ok) {
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t key = xk[row * 8 + jj];
        const int e = xi[row * 8 + jj];
        if (key > tk[7] && e >= 0 && e < args.E) topk_insert(tk, ti, key, e);
      }
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    // drain what is in flight before the ring is reused and TMEM freed
    bool drained = true;
    if (warp == 0 && lane == 0) {
      for (int st = 0; st < ST; ++st)
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
  const bool ok_cta = !*abort_flag;
  cluster_sync();  // both CTAs' MMAs are complete: CTA 0's ring may be written

  const bool lister = warp >= 2 && ((warp - 2) >> 2) == 0;  // the half-0 warps hold the lists
  const int row = (warp & 3) * 32 + lane;
  if (rank == 1 && lister) {  // also after an abort: empty lists (key 0) merge nothing
    const uint32_t dk = mapa_shared(smem_u32(rk), 0) + static_cast<uint32_t>(row * 32);
    const uint32_t di = mapa_shared(smem_u32(ri), 0) + static_cast<uint32_t>(row * 32);
    st_cluster_v4(dk, __uint_as_float(tk[0]), __uint_as_float(tk[1]), __uint_as_float(tk[2]), __uint_as_float(tk[3]));
    st_cluster_v4(dk + 16, __uint_as_float(tk[4]), __uint_as_float(tk[5]), __uint_as_float(tk[6]),
                  __uint_as_float(tk[7]));
    st_cluster_v4(di, __int_as_float(ti[0]), __int_as_float(ti[1]), __int_as_float(ti[2]), __int_as_float(ti[3]));
    st_cluster_v4(di + 16, __int_as_float(ti[4]), __int_as_float(ti[5]), __int_as_float(ti[6]), __int_as_float(ti[7]));
  }
  cluster_sync();  // CTA 1's lists have arrived

  if (rank == 0 && lister) {
    // (after an abort in CTA 1 the rows keep CTA 0's experts only; CTA 1's
    // status bit reports it)
    const int t = m0 + row;
    if (ok_cta && t < args.T) {
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        // an expert index outside [0, E) can only come from an aborted
        // partner's stale ring bytes; it is never taken
        const uint32_t key = rk[row * 8 + jj];
        const int e = ri[row * 8 + jj];
        if (key > tk[7] && e >= 0 && e < args.E) topk_insert(tk, ti, key, e);
      }
      write_row_topk(args, t, tk, ti);
    }
  }
  if (warp == 1 && !*drain_failed) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int NB>
constexpr int router_stages() {
  return (kRTileBytes * (1 + NB) * 4 <= 200 * 1024) ? 4 : ((kRTileBytes * (1 + NB) * 3 <= 200 * 1024) ? 3 : 2);
}
template <int NB>
constexpr size_t router_smem() {
  return 1024 + static_cast<size_t>(router_stages<NB>()) * kRTileBytes * (1 + NB) +
         (2 * router_stages<NB>() + 2) * 8 + 16;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [rows][H] bf16 row-major matrix, loaded in boxes of 64 elements x
// box_rows rows with the 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t H, int box_rows = kRM) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRKElems), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NB>
cudaError_t launch_nb(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, cudaStream_t stream) {
  constexpr int ST = router_stages<NB>();
  constexpr size_t smem = router_smem<NB>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(router_topk_kernel<NB, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return attr_err;
  const dim3 grid(static_cast<unsigned>((a.T + kRM - 1) / kRM));
  return launch_pdl(router_topk_kernel<NB, ST>, grid, dim3(kRThreads), smem, stream, mx, mw, a);
}

template <int NC>
constexpr int pair_stages() {
  return (200 * 1024) / (kRTileBytes + 32 * NC * 128) > 6 ? 6 : (200 * 1024) / (kRTileBytes + 32 * NC * 128);
}
template <int NC>
cudaError_t launch_pair(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, cudaStream_t stream) {
  constexpr int ST = pair_stages<NC>();
  constexpr size_t smem = 1024 + static_cast<size_t>(ST) * (kRTileBytes + 32 * NC * 128) + (2 * ST + 2) * 8 + 16;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(router_pair_kernel<NC, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.T + kRM - 1) / kRM * 2));
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, router_pair_kernel<NC, ST>, mx, mw, a);
}

template <int NB, int KS>
cudaError_t launch_split(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, cudaStream_t stream) {
  constexpr int ST = router_stages<NB>();
  constexpr size_t smem = router_smem<NB>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(router_split_kernel<NB, ST, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.T + kRM - 1) / kRM * KS));
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, router_split_kernel<NB, ST, KS>, mx, mw, a);
}

template <int NB>
cudaError_t launch_any(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, int ks,
                       cudaStream_t stream) {
  switch (ks) {
    case 4: return launch_split<NB, 4>(mx, mw, a, stream);
    case 8: return launch_split<NB, 8>(mx, mw, a, stream);
    default: return launch_nb<NB>(mx, mw, a, stream);
  }
}

// K split of the scores: 8 or 4 (each owner CTA ranking at most 32 rows) when
// it divides the k tiles and keeps the clusters within one wave of CTAs (148
// SMs, one CTA each); 1 (no split) for larger batches, where the unsplit
// kernel already fills the GPU and a 2-way split's per-row ranking costs more
// than it saves (measured: 101 us for 8192 tokens split in two against 73 us
// unsplit for 16384), and for 512 experts, whose receive slots would not fit
// in the ring.
int router_split(int T, int H, int nb) {
  if (nb > 3) return 1;
  const int m = (T + kRM - 1) / kRM, kt = H / kRKElems;
  for (int ks = 8; ks >= 4; ks >>= 1)
    if (kt % ks == 0 && m * ks <= 148) return ks;
  return 1;
}

}  // namespace

cudaError_t launch_router_topk(const void* x, const void* w_router, float* logits_out, int T, int E, int H, int k,
                               int32_t* topk_ids, float* topk_w, void* workspace, uint32_t* status,
                               cudaStream_t stream) {
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, T, H) || !make_map(&mw, w_router, E, H)) return cudaErrorInvalidValue;
  RouterArgs a;
  a.logits_out = logits_out;
  a.topk_ids = topk_ids;
  a.topk_w = topk_w;
  a.bitmap = route_small(T, E) ? nullptr : static_cast<uint32_t*>(workspace);  // small batches: no bitmaps here
  a.status = status;
  a.T = T;
  a.E = E;
  a.H = H;
  a.k = k;
  a.W = (T + 31) / 32;
  const int nb = (E + 127) / 128;
  const int ks = router_split(T, H, nb);
  // Mid-size batches (row tiles too many for the K split but fewer than one
  // per pair of SMs): the experts split over a two-CTA cluster, each CTA
  // streaming half of W_r.
  const int m_tiles = (T + kRM - 1) / kRM;
  if (ks == 1 && E % 128 == 0 && 2 * m_tiles <= 148) {
    CUtensorMap mwh;
    if (!make_map(&mwh, w_router, E, H, E / 2)) return cudaErrorInvalidValue;
    switch (E / 64) {
      case 2: return launch_pair<2>(mx, mwh, a, stream);
      case 4: return launch_pair<4>(mx, mwh, a, stream);
      case 6: return launch_pair<6>(mx, mwh, a, stream);
      case 8: return launch_pair<8>(mx, mwh, a, stream);
      default: break;
    }
  }
  switch (nb) {
    case 1: return launch_any<1>(mx, mw, a, ks, stream);
    case 2: return launch_any<2>(mx, mw, a, ks, stream);
    case 3: return launch_any<3>(mx, mw, a, ks, stream);
    case 4: return launch_nb<4>(mx, mw, a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
