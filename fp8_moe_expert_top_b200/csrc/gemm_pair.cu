// The grouped block-scaled GEMMs on SM pairs (selected with
// MOE_B200_GEMM=pair; the one-SM kernel of gemm.cu is the default).
//
// Same computation and epilogue as the one-SM kernel; the difference is how a
// tile's operands reach the tensor cores.  A pair of CTAs (a cluster of two,
// one per SM) owns a 256-row x 256-column output tile of one expert: each CTA
// loads its own 128 activation rows and one half (128 rows) of the 256-row
// weight tile, plus the scales, and the leader CTA issues
// tcgen05.mma.cta_group::2 (M = 256), which reads the weight halves from both
// CTAs' shared memory.  A stage is 38 KB per SM instead of 54 KB for the same
// tensor-core work.  Measured at prefill it is bit-exact but about 1.7x slower
// per SM than the one-SM kernel: every MMA of the pair still needs its three
// scale-atom copies (cta_group::2) in each CTA's TMEM, and the leader's MMA
// thread spends most of its time waiting for them or blocked issuing.
//
// Synchronization: both CTAs' loads of a stage complete on the leader's
// "full" barrier (cp.async.bulk.tensor .cta_group::2, no multicast), on which
// each CTA's producer arrives once announcing its own bytes (the follower's
// arrival is remote), so neither waits for the other before loading; the
// MMA warp's commits arrive on the "empty" and "accumulator full" barriers of
// both CTAs (tcgen05.commit multicast); both CTAs' epilogue threads release the
// accumulator on the leader's "accumulator empty" barrier.  The leader's six
// copier warps move each stage's scale atoms into both CTAs' TMEM
// (tcgen05.cp.cta_group::2).  Every wait is bounded; a wait that runs out
// raises the abort flags of both CTAs, work in flight is drained, and a
// status bit is set.
#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "pair.cuh"
#include "quant.cuh"

namespace moe {

namespace {

constexpr int kPairStages = 5;
// Warp roles as in the one-SM kernel: warp 0 producer (both CTAs), warp 1
// MMA issuer (leader), warps 2-7 scale copiers (leader), warps 8-15 epilogue
// (both CTAs); registers 72 for warps 0-7, 184 for the epilogue warpgroups.
constexpr int kPairCopierWarps = 6;
constexpr int kPairEpiWarp0 = 2 + kPairCopierWarps;
constexpr int kPairThreads = 32 * (kPairEpiWarp0 + kEpiWarps);
constexpr uint32_t kPairRegsLight = 72;
constexpr uint32_t kPairRegsEpilogue = 184;
static_assert(kPairThreads == 512 && kPairEpiWarp0 % 4 == 0, "warpgroup-aligned roles");
static_assert(32 * kPairEpiWarp0 * kPairRegsLight + 32 * kEpiWarps * kPairRegsEpilogue <= 65536u,
              "the register split must fit in the block's launch allocation (512 x 128)");
template <int FMT>
constexpr uint32_t kPairSfCols = (FMT == MOE_NVFP4) ? 48u : 12u;  // TMEM scale columns per stage
static_assert(kBN + kPairStages * 48 <= kTmemCols, "scale buffers do not fit in TMEM");

// Every operand buffer is viewed as a 2-D array of 256-byte lines (the codes
// are stored pre-swizzled), so each copy is one box of whole lines.
constexpr int kLine = 256;

struct PairMaps {
  CUtensorMap a[4];  // activation codes, boxes of 32, 64, 96 and 128 rows of one tile (4..16 KB)
  CUtensorMap b;     // weight codes, box = half of a 256-row tile (16 KB)
  CUtensorMap asf1;  // activation scales, box = one 512-byte atom
  CUtensorMap asf4;  // box = four atoms (2 KB)
  CUtensorMap bsf1;  // weight scales, box = one atom
  CUtensorMap bsf4;  // box = four atoms
};

struct PairCoord {
  int e, we, nt, mt0;  // row group, its weight expert, weight tile, first of the pair's two row blocks
  bool bad;
};

// rows of a 128-row block that a CTA loads: the valid rows rounded up to 32
__device__ __forceinline__ int rows_loaded(int valid) { return valid <= 0 ? 0 : (valid + 31) / 32 * 32; }

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(kPairThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ PairMaps maps, const GemmArgs args) {
  using Tr = GemmTraits<FMT, 128, kPairStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kPairStages * Tr::kStageBytes);
  uint64_t* empty_bar = full_bar + kPairStages;
  uint64_t* tfull_bar = empty_bar + kPairStages;
  uint64_t* tempty_bar = tfull_bar + 1;
  uint64_t* sf_bar = tempty_bar + 1;           // a stage's scale copies are issued
  uint64_t* drain_bar = sf_bar + kPairStages;  // after an abort: the leader's tcgen05 work has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int32_t* s_offsets = reinterpret_cast<int32_t*>(tmem_slot + 4);
  int32_t* s_pstart = s_offsets + args.E + 1;  // first pair-tile of each row group

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full_bar[s], 2);  // one arrival per CTA of the pair
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_bar[s], kPairCopierWarps);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 2 * 32 * kEpiWarps);
    mbar_init(drain_bar, 1 + kPairCopierWarps);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&maps.a[i]);
    prefetch_tensormap(&maps.b);
    prefetch_tensormap(&maps.asf1);
    prefetch_tensormap(&maps.asf4);
    prefetch_tensormap(&maps.bsf1);
    prefetch_tensormap(&maps.bsf4);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();
  pdl_trigger();
  const int n_tiles = args.n_rows_b / kBN;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_offsets[i] = args.offsets[i];
  __syncthreads();
  if (warp == 0) {  // s_pstart[e] = sum over e' < e of pairs(e') * n_tiles
    int32_t carry = 0;
    for (int base = 0; base <= E; base += 32) {
      const int e = base + lane;
      int32_t v = 0;
      if (e < E) v = ((s_offsets[e + 1] - s_offsets[e]) / kBM + 1) / 2 * n_tiles;
      int32_t incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e <= E) s_pstart[e] = carry + incl - v;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialized before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = s_pstart[E];
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int k_tiles = (args.K + Tr::kElemsPerStage - 1) / Tr::kElemsPerStage;
  const int ktiles_row = static_cast<int>(args.kb >> 7);
  uint32_t fail_bits = 0;
  uint32_t armed = 0u, armed_par = 0u;

  auto coord = [&](int tile) {
    PairCoord c;
    int lo = 0, hi = E;  // s_pstart[lo] <= tile < s_pstart[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pstart[mid] <= tile) lo = mid;
      else hi = mid;
    }
    c.e = lo;
    const int pairs = ((s_offsets[lo + 1] - s_offsets[lo]) / kBM + 1) / 2;
    const int local = tile - s_pstart[lo];
    c.nt = local / pairs;
    c.mt0 = s_offsets[lo] / kBM + 2 * (local % pairs);
    c.we = c.e;
    c.bad = false;
    if (args.expert_map != nullptr) {
      const int w = __ldg(args.expert_map + c.e);
      c.bad = w < 0 || w >= args.n_weights;
      c.we = c.bad ? 0 : w;
    }
    return c;
  };

  // Roles by warpgroup (every warp of a warpgroup executes the same setmaxnreg).
  if (warp < kPairEpiWarp0) {
    reg_dealloc<kPairRegsLight>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      if (lane == 0) {
        const uint64_t pol_stream = policy_evict_first();
        const uint64_t pol_keep = policy_evict_normal();
        const uint64_t pol_a = policy_evict_last();
        const uint32_t full_leader0 = mapa_shared(smem_u32(&full_bar[0]), 0);
        int stage = 0;
        uint32_t phase = 0;
        for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
          const PairCoord c = coord(tile);
          const int e = c.e, we = c.we;
          const int rows_end = s_offsets[e] + __ldg(args.counts + e);
          const int v0 = max(0, min(kBM, rows_end - c.mt0 * kBM));
          const int v1 = max(0, min(kBM, rows_end - (c.mt0 + 1) * kBM));
          const int my_rows = rows_loaded(rank ? v1 : v0);
          const int my_mt = c.mt0 + static_cast<int>(rank);
          const uint64_t pol_w = (s_offsets[e + 1] - s_offsets[e]) > 2 * kBM ? pol_keep : pol_stream;
          // byte offsets of this CTA's k-tile 0 (tiles are 128 bytes wide, K tile fastest)
          const int64_t a_off0 = static_cast<int64_t>(my_mt) * ktiles_row * (kBM * 128);
          const int64_t b_off0 = (static_cast<int64_t>(we) * n_tiles + c.nt) * ktiles_row * (kBN * 128) +
                                 static_cast<int64_t>(kBM * 128) * rank;
          // a CTA whose row block holds no valid row (past its group, possibly
          // past the buffer) loads no codes, and the scales of the pair's first
          // block (its output rows are never stored)
          const int64_t asf0 = static_cast<int64_t>(my_rows > 0 ? my_mt : c.mt0) * args.sf_rb_stride;
          const int64_t bsf0 = static_cast<int64_t>(we) * args.b_sf_expert_stride +
                               static_cast<int64_t>(c.nt) * (kBN / 128) * args.sf_rb_stride;
          for (int kt = 0; kt < k_tiles; ++kt) {
            if (!mbar_wait_pair(&empty_bar[stage], phase ^ 1u, abort_flag, peer_abort)) {
              fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
              break;
            }
            const int kb_here = min(4, (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK);
            const int atoms = (FMT == MOE_NVFP4) ? kb_here : 1;
            const uint32_t sf_bytes = 512u * atoms;
            const uint32_t bar = full_leader0 + 8u * stage;
            // this CTA's bytes of the stage: its activation rows, its half of
            // the weight tile, the activation scales and both weight halves' scales
            const uint32_t my_bytes = static_cast<uint32_t>(my_rows) * 128u + 16384u + 3u * sf_bytes;
            if (leader) {
              mbar_arrive_expect_tx(&full_bar[stage], my_bytes);
              armed |= 1u << stage;
              armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            } else {
              // the previous phase of this stage completed before the MMAs that
              // freed it ran, so this arrival belongs to the phase being filled
              mbar_arrive_expect_tx_cluster(bar, my_bytes);
            }
            uint8_t* st = smem + stage * Tr::kStageBytes;
            const int64_t a_off = a_off0 + static_cast<int64_t>(kt) * (kBM * 128);
            if (my_rows > 0)
              tma_load_2d_pair(st, &maps.a[my_rows / 32 - 1], 0, static_cast<int32_t>(a_off / kLine), bar, pol_a);
            tma_load_2d_pair(st + Tr::kABytes, &maps.b, 0,
                             static_cast<int32_t>((b_off0 + static_cast<int64_t>(kt) * (kBN * 128)) / kLine), bar,
                             pol_w);
            const int64_t asf_off = asf0 + static_cast<int64_t>(kt) * Tr::kSfBytes128;
            if (atoms == 4) {
              tma_load_2d_pair(st + Tr::kSfaOff, &maps.asf4, 0, static_cast<int32_t>(asf_off / kLine), bar, pol_a);
            } else {
              for (int a = 0; a < atoms; ++a)
                tma_load_2d_pair(st + Tr::kSfaOff + 512 * a, &maps.asf1, 0,
                                 static_cast<int32_t>((asf_off + 512 * a) / kLine), bar, pol_a);
            }
  #pragma unroll
            for (int h = 0; h < kBN / 128; ++h) {
              const int64_t bsf_off = bsf0 + h * args.sf_rb_stride + static_cast<int64_t>(kt) * Tr::kSfBytes128;
              uint8_t* dst = st + Tr::kSfbOff + h * Tr::kSfBytes128;
              if (atoms == 4) {
                tma_load_2d_pair(dst, &maps.bsf4, 0, static_cast<int32_t>(bsf_off / kLine), bar, pol_w);
              } else {
                for (int a = 0; a < atoms; ++a)
                  tma_load_2d_pair(dst + 512 * a, &maps.bsf1, 0, static_cast<int32_t>((bsf_off + 512 * a) / kLine),
                                   bar, pol_w);
              }
            }
            if (++stage == kPairStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (leader)
      if (lane == 0 && leader) {
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0;
        const uint32_t d_tmem = tmem_base;
        for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
          if (!mbar_wait_pair(tempty_bar, acc_phase ^ 1u, abort_flag, peer_abort)) {
            fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
            break;
          }
          tc_fence_after();
          bool ok = true;
          for (int kt = 0; kt < k_tiles; ++kt) {
            if (!mbar_wait_pair(&sf_bar[stage], phase, abort_flag, peer_abort) ||
                !mbar_wait_pair(&full_bar[stage], phase, abort_flag, peer_abort)) {
              fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
              ok = false;
              break;
            }
            tc_fence_after();
            const int kb_here = min(4, (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK);
            const uint32_t st = smem_u32(smem + stage * Tr::kStageBytes);
            const uint64_t adesc = make_desc_sw128(st);
            const uint64_t bdesc = make_desc_sw128(st + Tr::kABytes);
            const uint32_t sfa = tmem_base + Tr::kTmemSfa + stage * kPairSfCols<FMT>;
            const uint32_t sfb = sfa + Tr::kSfaCols;
            if (FMT == MOE_NVFP4) {
              for (int kb = 0; kb < kb_here; ++kb)
                tc_mma_nvfp4_pair(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_nvfp4(kBN, 2 * kBM), sfa + 4 * kb,
                                  sfb + (kBN / 32) * kb, (kt | kb) != 0 ? 1u : 0u);
            } else {
              for (int kb = 0; kb < kb_here; ++kb) {
                const uint32_t sel = static_cast<uint32_t>(kb) << 30;
                tc_mma_mxfp8_pair(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_mxfp8(kBN, kb, 2 * kBM), sfa | sel,
                                  sfb | sel, (kt | kb) != 0 ? 1u : 0u);
              }
            }
            tc_commit_pair(&empty_bar[stage], 0x3);
            if (++stage == kPairStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit_pair(tfull_bar, 0x3);
          acc_phase ^= 1u;
        }
      }
    } else if (warp < kPairEpiWarp0) {
      // ------------------------------------------------------------ scale copiers (leader)
      // Copier c moves atoms c and c + 6 of an NVFP4 stage (atom j: k block
      // j / 3; the A atom or weight half j % 3 - 1), atom c of an MXFP8 stage,
      // of each CTA into its own TMEM (cta_group::2), into the stage's columns,
      // last read by the MMAs of the same stage one ring turn ago (complete
      // before the stage was freed and refilled, i.e. before the full barrier
      // below completes).
      const int cp = warp - 2;
      if (lane == 0 && leader) {
        int stage = 0;
        uint32_t phase = 0;
        for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
          bool ok = true;
          for (int kt = 0; kt < k_tiles; ++kt) {
            if (!mbar_wait_pair(&full_bar[stage], phase, abort_flag, peer_abort)) {
              fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
              ok = false;
              break;
            }
            tc_fence_after();
            const int kb_here = min(4, (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK);
            const uint32_t st = smem_u32(smem + stage * Tr::kStageBytes);
            const uint32_t sfa = tmem_base + Tr::kTmemSfa + stage * kPairSfCols<FMT>;
            const uint32_t sfb = sfa + Tr::kSfaCols;
            if (FMT == MOE_NVFP4) {
              for (int j = cp; j < 3 * kb_here; j += kPairCopierWarps) {
                const int kb = j / 3, m = j % 3;
                if (m == 0)
                  tc_cp_sf_atom_pair(sfa + 4 * kb, make_desc_sf(st + Tr::kSfaOff + 512 * kb));
                else
                  tc_cp_sf_atom_pair(sfb + (kBN / 32) * kb + 4 * (m - 1),
                                     make_desc_sf(st + Tr::kSfbOff + (m - 1) * Tr::kSfBytes128 + 512 * kb));
              }
            } else if (cp == 0) {
              tc_cp_sf_atom_pair(sfa, make_desc_sf(st + Tr::kSfaOff));
            } else if (cp < 3) {
              tc_cp_sf_atom_pair(sfb + 4 * (cp - 1), make_desc_sf(st + Tr::kSfbOff + (cp - 1) * Tr::kSfBytes128));
            }
            // issued, not completed: copy -> MMA is a pipelined pair (see gemm.cu)
            tc_fence_before();
            mbar_arrive(&sf_bar[stage]);
            if (++stage == kPairStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
        }
      }
    }
  } else {
    reg_alloc<kPairRegsEpilogue>();
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - kPairEpiWarp0) >> 2;
    const int row_l = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + half * (kBN / 2);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty_bar), 0);
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
      const PairCoord c = coord(tile);
      const int e = c.e;
      const int64_t row = static_cast<int64_t>(c.mt0 + static_cast<int>(rank)) * kBM + row_l;
      const bool valid = row < s_offsets[e] + __ldg(args.counts + e);
      if (c.bad && warp == 2 && lane == 0) fail_bits |= MOE_DEVICE_BAD_GROUP_EXPERT;
      if (!mbar_wait_pair(tfull_bar, acc_phase, abort_flag, peer_abort)) {
        fail_bits |= MOE_DEVICE_TIMEOUT_EPILOGUE;
        break;
      }
      tc_fence_after();
      float acc[kBN / 2];
#pragma unroll
      for (int j = 0; j < kBN / 64; ++j) tmem_ld32(t_row + 32 * j, acc + 32 * j);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader);
      acc_phase ^= 1u;
      if (!valid) continue;
      epilogue_rows<FMT, GATEUP>(args, acc, row, c.we, c.nt, half);
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' roles are done: the abort flags no longer change
  tc_fence_after();
  if (*abort_flag) {
    // drain what the leader issued: the pair's copies complete on its full
    // barriers; its MMAs and scale copies on the drain barrier
    bool drained = true;
    if (leader && warp == 0 && lane == 0) {
      for (int st = 0; st < kPairStages; ++st)
        if ((armed >> st) & 1u) drained = mbar_wait_drain_cluster(&full_bar[st], (armed_par >> st) & 1u) && drained;
    } else if (leader && warp >= 1 && warp < kPairEpiWarp0 && lane == 0) {
      tc_commit_pair(drain_bar, 0x1);
      drained = mbar_wait_drain_cluster(drain_bar, 0);
    } else if (!leader && warp == 0 && lane == 0) {
      // copies this CTA issued into a phase the leader never arrived on
      // complete on no barrier anyone waits for: give them time to land (a
      // bulk copy of one stage takes microseconds) before the CTA can exit
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 50000u) {
      }
    }
    if (!drained) {
      *drain_failed = 1;
      st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(drain_failed)), 1u), 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair is done with each other's shared memory and TMEM
  tc_fence_after();
  if (warp == 1 && !*drain_failed) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point.
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

// A buffer of `bytes` bytes viewed as lines of kLine bytes; box = `box_bytes`
// (a multiple of kLine) of consecutive lines.
bool make_line_map(CUtensorMap* map, const void* base, int64_t bytes, int box_bytes) {
  if (bytes % kLine != 0 || box_bytes % kLine != 0 || box_bytes / kLine > 256) return false;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kLine), static_cast<cuuint64_t>(bytes / kLine)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kLine)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLine), static_cast<cuuint32_t>(box_bytes / kLine)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, bool GATEUP>
size_t pair_smem(int E) {
  using Tr = GemmTraits<FMT, 128, kPairStages>;
  return 1024 + kPairStages * Tr::kStageBytes + (3 * kPairStages + 3) * 8 + 16 + 2 * (E + 1) * 4;
}

template <int FMT, bool GATEUP>
cudaError_t launch_pair_one(const PairMaps& maps, const GemmArgs& a, cudaStream_t stream) {
  const size_t smem_max = pair_smem<FMT, GATEUP>(1024);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // per device: the shared-memory limit raised and the co-resident cluster
  // count read once
  static std::atomic<int> clusters[64];
  int n = clusters[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    err = cudaFuncSetAttribute(moe_gemm_pair_kernel<FMT, GATEUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_max));
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2);
    qc.blockDim = dim3(kPairThreads);
    qc.dynamicSmemBytes = smem_max;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.attrs = qa;
    qc.numAttrs = 1;
    err = cudaOccupancyMaxActiveClusters(&n, moe_gemm_pair_kernel<FMT, GATEUP>, &qc);
    if (err != cudaSuccess) return err;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    clusters[dev].store(n, std::memory_order_relaxed);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * n);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = pair_smem<FMT, GATEUP>(a.E);
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
  return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel<FMT, GATEUP>, maps, a);
}

}  // namespace

cudaError_t launch_gemm_pair(const GemmLaunch& g, const GemmArgs& a, cudaStream_t stream) {
  const int bits = (g.fmt == MOE_NVFP4) ? 4 : 8;
  const int sfvec = (g.fmt == MOE_NVFP4) ? 16 : 32;
  const int64_t kb = kb_padded(g.K, bits);
  const int64_t a_bytes = g.R_max * kb;
  const int64_t b_bytes = static_cast<int64_t>(a.n_weights) * g.n_rows_b * kb;
  const int64_t asf_bytes = g.R_max * (g.K / sfvec);
  const int64_t bsf_bytes = static_cast<int64_t>(a.n_weights) * g.n_rows_b * (g.K / sfvec);
  PairMaps m;
  for (int i = 0; i < 4; ++i)
    if (!make_line_map(&m.a[i], g.a_codes, a_bytes, 32 * (i + 1) * 128)) return cudaErrorInvalidValue;
  if (!make_line_map(&m.b, g.b_codes, b_bytes, kBM * 128) || !make_line_map(&m.asf1, g.a_sf, asf_bytes, 512) ||
      !make_line_map(&m.asf4, g.a_sf, asf_bytes, 2048) || !make_line_map(&m.bsf1, g.b_sf, bsf_bytes, 512) ||
      !make_line_map(&m.bsf4, g.b_sf, bsf_bytes, 2048))
    return cudaErrorInvalidValue;
  if (g.fmt == MOE_NVFP4)
    return g.gateup ? launch_pair_one<MOE_NVFP4, true>(m, a, stream) : launch_pair_one<MOE_NVFP4, false>(m, a, stream);
  return g.gateup ? launch_pair_one<MOE_MXFP8, true>(m, a, stream) : launch_pair_one<MOE_MXFP8, false>(m, a, stream);
}

}  // namespace moe
