// The grouped block-scaled GEMM on SM pairs (cluster of two CTAs), for
// batches whose experts hold several 128-row blocks (prefill).
//
// Same computation and epilogue as the one-SM kernel in gemm.cu; the
// difference is how a tile's operands reach the tensor cores.  A pair owns a
// 256-row x 256-column output tile of one expert: each CTA loads its own 128
// activation rows and one half (128 rows) of the 256-row weight tile, plus
// all scales, and the even CTA issues tcgen05.mma.cta_group::2 (M = 256),
// which reads the weight halves from both CTAs' shared memory.  Per SM a
// stage is 38 KB instead of 54 KB, so five stages fit and each byte brought
// into shared memory feeds twice the tensor work.
//
// Synchronization: all loads of a stage (both CTAs) complete on the even
// CTA's "full" barrier (cp.async.bulk.tensor .cta_group::2, no multicast);
// the MMA warp's commits arrive on the "empty" and "accumulator full"
// barriers of both CTAs (tcgen05.commit multicast); both CTAs' epilogue
// threads release the accumulator on the even CTA's "accumulator empty"
// barrier.  Scale atoms reach TMEM as in gemm.cu (per-stage columns, copied
// by two copier warps of the even CTA with tcgen05.cp.cta_group::2).  Waits
// are bounded as in gemm.cu.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {

constexpr int kPairStages = 5;
constexpr int kCopierWarps = 2;  // scale-copier warps (even CTA)
constexpr int kPairThreads = kThreads + 32 * kCopierWarps;
template <int FMT>
constexpr uint32_t kPairSfCols = (FMT == MOE_NVFP4) ? 48u : 12u;  // TMEM scale columns per stage
static_assert(kBN + kPairStages * 48 <= kTmemCols, "scale buffers do not fit in TMEM");

// Every operand buffer is viewed as a 2-D array of lines (no swizzle: the
// codes are stored pre-swizzled), so that each copy below is one box of whole
// lines.  Wide lines keep the number of box rows the copy engine walks per
// stage small.
constexpr int kCodeLine = 256;  // bytes per line of the code buffers
constexpr int kSfLine = 256;    // bytes per line of the scale buffers

struct PairMaps {
  CUtensorMap a_full;  // activation codes, box = one 128-row x 128-B tile (16 KB)
  CUtensorMap a_part;  // same buffer, box = 16 rows of a tile (2 KB)
  CUtensorMap b;       // weight codes, box = half of a 256-row tile (16 KB)
  CUtensorMap asf1;    // activation scales, box = one 512-B atom
  CUtensorMap asf4;    // box = four atoms (2 KB)
  CUtensorMap bsf1;    // weight scales, box = one atom
  CUtensorMap bsf4;    // box = four atoms
};

struct PairCoord {
  int e, nt, mt0;  // expert, weight tile, first of the pair's two row blocks
};

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
  uint64_t* sf_bar = tempty_bar + 1;  // a stage's scales are in both CTAs' TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_bar + kPairStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_offsets = reinterpret_cast<int32_t*>(tmem_slot + 4);
  int32_t* s_pstart = s_offsets + args.E + 1;  // first pair-tile of each expert

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_bar[s], kCopierWarps);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 2 * 32 * kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    prefetch_tensormap(&maps.a_full);
    prefetch_tensormap(&maps.a_part);
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
    return c;
  };

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
        const int e = c.e;
        const int rows_end = s_offsets[e] + __ldg(args.counts + e);
        const int v0 = max(0, min(kBM, rows_end - c.mt0 * kBM));
        const int v1 = max(0, min(kBM, rows_end - (c.mt0 + 1) * kBM));
        const int my_valid = rank ? v1 : v0;
        const int my_mt = c.mt0 + static_cast<int>(rank);
        const uint64_t pol_w = (s_offsets[e + 1] - s_offsets[e]) > 2 * kBM ? pol_keep : pol_stream;
        // byte offsets of this CTA's k-tile 0 (tiles are 128 B wide, K tile fastest)
        const int64_t a_off0 = static_cast<int64_t>(my_mt) * ktiles_row * (kBM * 128);
        const int64_t b_off0 = (static_cast<int64_t>(e) * n_tiles + c.nt) * ktiles_row * (kBN * 128) +
                               static_cast<int64_t>(kBM * 128) * rank;
        // a CTA whose row block holds no valid row (past the expert, possibly
        // past the buffer) still fills its scale slot, from the pair's first block
        const int64_t asf0 = static_cast<int64_t>(my_valid > 0 ? my_mt : c.mt0) * args.sf_rb_stride;
        const int64_t bsf0 = static_cast<int64_t>(e) * args.b_sf_expert_stride +
                             static_cast<int64_t>(c.nt) * (kBN / 128) * args.sf_rb_stride;
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
            fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
            break;
          }
          const int kb_here = min(4, (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK);
          const int atoms = (FMT == MOE_NVFP4) ? kb_here : 1;
          const uint32_t sf_bytes = 512u * atoms;
          const uint32_t bar = full_leader0 + 8u * stage;
          if (leader) {
            const uint32_t a_bytes = static_cast<uint32_t>((v0 + 15) / 16 + (v1 + 15) / 16) * 16 * kRowBytesPerStage;
            mbar_arrive_expect_tx(&full_bar[stage], a_bytes + 2u * (Tr::kBBytes + 3u * sf_bytes));
          }
          uint8_t* st = smem + stage * Tr::kStageBytes;
          auto line = [](int64_t byte_off) { return static_cast<int32_t>(byte_off / kCodeLine); };
          auto sf_line = [](int64_t byte_off) { return static_cast<int32_t>(byte_off / kSfLine); };
          const int64_t a_off = a_off0 + static_cast<int64_t>(kt) * (kBM * 128);
          if (my_valid == kBM) {
            tma_load_2d_pair(st, &maps.a_full, 0, line(a_off), bar, pol_a);
          } else {
            for (int i = 0; i < (my_valid + 15) / 16; ++i)
              tma_load_2d_pair(st + i * 16 * kRowBytesPerStage, &maps.a_part, 0, line(a_off + i * 16 * 128), bar,
                               pol_a);
          }
          tma_load_2d_pair(st + Tr::kABytes, &maps.b, 0, line(b_off0 + static_cast<int64_t>(kt) * (kBN * 128)), bar,
                           pol_w);
          const int64_t asf_off = asf0 + static_cast<int64_t>(kt) * Tr::kSfBytes128;
          if (atoms == 4) {
            tma_load_2d_pair(st + Tr::kSfaOff, &maps.asf4, 0, sf_line(asf_off), bar, pol_a);
          } else {
            for (int a = 0; a < atoms; ++a)
              tma_load_2d_pair(st + Tr::kSfaOff + 512 * a, &maps.asf1, 0, sf_line(asf_off + 512 * a), bar, pol_a);
          }
#pragma unroll
          for (int h = 0; h < kBN / 128; ++h) {
            const int64_t bsf_off = bsf0 + h * args.sf_rb_stride + static_cast<int64_t>(kt) * Tr::kSfBytes128;
            uint8_t* dst = st + Tr::kSfbOff + h * Tr::kSfBytes128;
            if (atoms == 4) {
              tma_load_2d_pair(dst, &maps.bsf4, 0, sf_line(bsf_off), bar, pol_w);
            } else {
              for (int a = 0; a < atoms; ++a)
                tma_load_2d_pair(dst + 512 * a, &maps.bsf1, 0, sf_line(bsf_off + 512 * a), bar, pol_w);
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
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t d_tmem = tmem_base;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        if (!mbar_wait<true>(tempty_bar, acc_phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait<true>(&sf_bar[stage], phase, abort_flag) ||
              !mbar_wait<true>(&full_bar[stage], phase, abort_flag)) {
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
            for (int kb = 0; kb < kb_here; ++kb) {
              tc_mma_nvfp4_pair(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_nvfp4(kBN, 2 * kBM), sfa + 4 * kb,
                                sfb + (kBN / 32) * kb, (kt | kb) != 0 ? 1u : 0u);
            }
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
  } else if (warp >= kThreads / 32) {
    // ------------------------------------------------------------ scale copiers (even CTA)
    // Copy each CTA's scale atoms of every kCopierWarps-th k block into its
    // own TMEM (cta_group::2), into the stage's own columns, and signal the MMA
    // thread.  The columns were last read by the MMAs of the same stage one
    // ring turn ago, which completed before the stage was released and refilled.
    const int part = warp - kThreads / 32;
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait<true>(&full_bar[stage], phase, abort_flag)) {
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
            for (int kb = part; kb < kb_here; kb += kCopierWarps) {
              tc_cp_sf_atom_pair(sfa + 4 * kb, make_desc_sf(st + Tr::kSfaOff + 512 * kb));
#pragma unroll
              for (int h = 0; h < kBN / 128; ++h)
                tc_cp_sf_atom_pair(sfb + (kBN / 32) * kb + 4 * h,
                      make_desc_sf(st + Tr::kSfbOff + h * Tr::kSfBytes128 + 512 * kb));
            }
          } else if (part == 0) {
            tc_cp_sf_atom_pair(sfa, make_desc_sf(st + Tr::kSfaOff));
            tc_cp_sf_atom_pair(sfb, make_desc_sf(st + Tr::kSfbOff));
          } else {
#pragma unroll
            for (int h = 1; h < kBN / 128; ++h)
              tc_cp_sf_atom_pair(sfb + 4 * h, make_desc_sf(st + Tr::kSfbOff + h * Tr::kSfBytes128));
          }
          tc_commit_pair(&sf_bar[stage], 0x1);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_l = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + half * (kBN / 2);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty_bar), 0);
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
      const PairCoord c = coord(tile);
      const int e = c.e;
      const int64_t row = static_cast<int64_t>(c.mt0 + static_cast<int>(rank)) * kBM + row_l;
      const bool valid = row < s_offsets[e] + __ldg(args.counts + e);
      if (!mbar_wait(tfull_bar, acc_phase, abort_flag)) {
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
      epilogue_rows<FMT, GATEUP>(args, acc, row, e, c.nt, half);
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair is done with each other's shared memory and TMEM
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// A buffer of `bytes` bytes viewed as lines of `width` bytes; box = `box_bytes`
// (a multiple of width) of consecutive lines.
static bool make_line_map(CUtensorMap* map, const void* base, int64_t bytes, int64_t width, int box_bytes) {
  if (bytes % width != 0 || box_bytes % width != 0 || box_bytes / width > 256) return false;
  const int64_t lines = bytes / width, box_lines = box_bytes / width;
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(lines)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(width)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(width), static_cast<cuuint32_t>(box_lines)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, bool GATEUP>
static cudaError_t launch_pair_one(const PairMaps& maps, const GemmArgs& a, cudaStream_t stream) {
  using Tr = GemmTraits<FMT, 128, kPairStages>;
  const size_t smem_max = 1024 + kPairStages * Tr::kStageBytes + (3 * kPairStages + 2) * 8 + 16 + 2 * 1025 * 4;
  const size_t smem = 1024 + kPairStages * Tr::kStageBytes + (3 * kPairStages + 2) * 8 + 16 + 2 * (a.E + 1) * 4;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  static int clusters[64] = {0};
  if (dev >= 64 || clusters[dev] == 0) {
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
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, moe_gemm_pair_kernel<FMT, GATEUP>, &qc);
    if (err != cudaSuccess) return err;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    if (dev < 64) clusters[dev] = n;
    else return cudaErrorInvalidDevice;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters[dev]);
  cfg.blockDim = dim3(kPairThreads);
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
  return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel<FMT, GATEUP>, maps, a);
}

cudaError_t launch_gemm_pair(const GemmLaunch& g, const GemmArgs& a, cudaStream_t stream) {
  const int bits = (g.fmt == MOE_NVFP4) ? 4 : 8;
  const int sfvec = (g.fmt == MOE_NVFP4) ? 16 : 32;
  const int64_t kb = kb_padded(g.K, bits);
  const int64_t a_bytes = g.R_max * kb;
  const int64_t b_bytes = static_cast<int64_t>(g.E) * g.n_rows_b * kb;
  const int64_t asf_bytes = g.R_max * (g.K / sfvec);
  const int64_t bsf_bytes = static_cast<int64_t>(g.E) * g.n_rows_b * (g.K / sfvec);
  PairMaps m;
  if (!make_line_map(&m.a_full, g.a_codes, a_bytes, kCodeLine, kBM * 128) ||
      !make_line_map(&m.a_part, g.a_codes, a_bytes, kCodeLine, 16 * 128) ||
      !make_line_map(&m.b, g.b_codes, b_bytes, kCodeLine, kBM * 128) ||
      !make_line_map(&m.asf1, g.a_sf, asf_bytes, kSfLine, 512) ||
      !make_line_map(&m.asf4, g.a_sf, asf_bytes, kSfLine, 2048) ||
      !make_line_map(&m.bsf1, g.b_sf, bsf_bytes, kSfLine, 512) ||
      !make_line_map(&m.bsf4, g.b_sf, bsf_bytes, kSfLine, 2048))
    return cudaErrorInvalidValue;
  if (g.fmt == MOE_NVFP4)
    return g.gateup ? launch_pair_one<MOE_NVFP4, true>(m, a, stream) : launch_pair_one<MOE_NVFP4, false>(m, a, stream);
  return g.gateup ? launch_pair_one<MOE_MXFP8, true>(m, a, stream) : launch_pair_one<MOE_MXFP8, false>(m, a, stream);
}

}  // namespace moe
