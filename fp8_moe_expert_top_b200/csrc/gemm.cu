// Persistent grouped block-scaled GEMMs of the expert FFN on tcgen05.
//
// Page "Thinking Machines releases Inkling 2 Small weights under Apache
// 2.0", section "NVFP4 and MXFP8 experts": every token is processed by 8 of
// 384 experts whose weights are NVFP4 (E2M1 with E4M3 block scales) or MXFP8
// (E4M3 with E8M0 block scales), and the activations are quantized to that
// format inside the kernel that produces them.  The gate/up GEMM therefore
// ends in an epilogue that applies SwiGLU and requantizes h in registers
// (NVFP4 with the 4-vs-6 pick of the section TL;DR), and the down GEMM reads
// those codes directly.
//
// Tiling: a tile is 128 permuted rows (one expert's segment is a whole
// number of 128-row blocks) x BN = 256 rows of that expert's weight matrix,
// with K streamed in steps of 128 bytes per row (256 NVFP4 or 128 MXFP8
// elements).  One CTA per SM walks the tile list (row block fastest-varying
// over N tiles, so the tiles sharing an activation block run together and
// the weight tiles of one expert are reused from L2 across its row blocks).
//
// Operands are stored pre-tiled and pre-swizzled (tiles of rows x 128 bytes,
// K tile fastest, the 128-byte swizzle applied in memory), so every stage is
// one contiguous 1-D bulk copy per operand.
//
// Warp roles (384 threads):
//   warp 0      producer: bulk copies of A, B and their scale atoms into a
//               4-stage ring
//   warp 1      MMA issuer: TMEM allocation, tcgen05.mma block-scaled
//               M=128 N=256, commits
//   warps 2-9   epilogue: tcgen05.ld of the 128x256 fp32 accumulator (two
//               warps per TMEM lane quarter, 128 columns each), tensor scales,
//               SwiGLU + requantization (gate/up) or bf16 store (down)
//   warps 10-11 scale copiers: the stage's scale atoms SMEM -> TMEM
//               (tcgen05.cp), alternate k blocks each, into per-stage TMEM
//               columns; they signal the MMA thread once the copies are
//               issued (the copy -> MMA order is kept by the tensor pipe).
// A tcgen05.cp holds its issuing thread for about 50 cycles and the copies
// share the tensor pipe with the MMAs; issued by the MMA thread they delay
// its MMAs (measured: the prefill gate/up GEMM 1.5x slower), so each stage's
// 12 (NVFP4) copies are spread over threads of their own.  A tcgen05.cp is
// issued once per warp instruction, not once per active lane: the issuing
// threads must be lanes of different warps.
// Every mbarrier wait is bounded; a wait that runs out raises a CTA-wide
// abort flag and every role stops issuing.  Work already in flight (bulk
// copies into stages nobody consumed, MMAs, scale copies) is then waited for,
// again with a time limit, before TMEM is freed; if that wait also runs out,
// TMEM is left allocated rather than freed under a running tensor-core
// operation.  A status bit reports the abort.
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {

constexpr int kStages = 4;
constexpr int kCopierWarps = 2;  // scale-copier warps
constexpr int kThreadsOne = kThreads + 32 * kCopierWarps;
// TMEM columns of one stage's scales: NVFP4 4 (A) + 8 (B) per 64-element k
// block x 4 k blocks; MXFP8 4 + 8 (one 32-bit column holds 4 k blocks)
template <int FMT>
constexpr uint32_t kSfColsPerStage = (FMT == MOE_NVFP4) ? 48u : 12u;
static_assert(kBN + kStages * 48 <= kTmemCols, "scale buffers do not fit in TMEM");
// Tile order: expert by expert; inside an expert, weight tile (nt) by weight
// tile, and the expert's 128-row blocks (mt) fastest.  CTAs running at the same
// time therefore share one weight tile (read from HBM once, then from L2), and
// an expert's activation rows are re-read from L2 for each weight tile.
// A row group is one expert's segment; with an expert map (grouped calls)
// group e uses the weights of expert map[e] (an index outside the packed
// weights is clamped to 0 and reported through the status word).
struct TileCoord {
  int e, we, mt, nt, m_blocks;
  bool bad;
};
__device__ __forceinline__ TileCoord tile_coord(int tile, const int32_t* offs, int E, int n_tiles,
                                                const int32_t* emap, int n_weights) {
  TileCoord c;
  c.e = find_expert(offs, E, (tile / n_tiles) * kBM);
  const int mt0 = offs[c.e] / kBM;
  c.m_blocks = offs[c.e + 1] / kBM - mt0;
  const int local = tile - mt0 * n_tiles;
  c.nt = local / c.m_blocks;
  c.mt = mt0 + local % c.m_blocks;
  c.we = c.e;
  c.bad = false;
  if (emap != nullptr) {
    const int w = __ldg(emap + c.e);
    c.bad = w < 0 || w >= n_weights;
    c.we = c.bad ? 0 : w;
  }
  return c;
}

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(kThreadsOne, 1)
    moe_gemm_kernel(const GemmArgs args) {
  using Tr = GemmTraits<FMT, kBN, kStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kStages * Tr::kStageBytes);
  uint64_t* empty_bar = full_bar + kStages;
  uint64_t* tfull_bar = empty_bar + kStages;
  uint64_t* tempty_bar = tfull_bar + 1;
  uint64_t* sf_bar = tempty_bar + 1;  // a stage's scale copies are issued
  uint64_t* drain_bar = sf_bar + kStages;  // after an abort: in-flight tcgen05 work has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_failed = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int32_t* s_offsets = reinterpret_cast<int32_t*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_bar[s], kCopierWarps);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 32 * kEpiWarps);
    mbar_init(drain_bar, 1 + kCopierWarps);
    *abort_flag = 0;
    *drain_failed = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // everything above overlaps the previous kernel; from here on its outputs are read
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_offsets[i] = args.offsets[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m_tiles = s_offsets[E] / kBM;
  const int n_tiles = args.n_rows_b / kBN;
  const int total = m_tiles * n_tiles;
  const int k_tiles = (args.K + Tr::kElemsPerStage - 1) / Tr::kElemsPerStage;
  uint32_t fail_bits = 0;
  // producer: stages armed for a bulk copy (bit s) and the full-barrier
  // phase parity each was armed in; drained after an abort
  uint32_t armed = 0u, armed_par = 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // weights read by a single row block are streamed once; otherwise they
      // are reused by the expert's other row blocks and stay in L2
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_normal();
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, s_offsets, E, n_tiles, args.expert_map, args.n_weights);
        const int mt = tc.mt, nt = tc.nt, e = tc.e, we = tc.we;
        const uint64_t pol_w = tc.m_blocks > 1 ? pol_keep : pol_stream;
        const uint8_t* a_sf = args.a_sf + static_cast<int64_t>(mt) * args.sf_rb_stride;
        const uint8_t* b_sf = args.b_sf + static_cast<int64_t>(we) * args.b_sf_expert_stride +
                              static_cast<int64_t>(nt) * (kBN / 128) * args.sf_rb_stride;
        const int64_t ktiles_row = args.kb >> 7;  // K tiles per code row
        const uint8_t* a_tiles = args.a_codes + static_cast<int64_t>(mt) * ktiles_row * Tr::kABytes;
        const uint8_t* b_tiles = args.b_codes + static_cast<int64_t>(we) * args.b_expert_stride +
                                 static_cast<int64_t>(nt) * ktiles_row * Tr::kBBytes;
        // Only the row block's valid rows are loaded (rounded up to 16); the
        // rest of the A tile keeps stale data, whose output rows are never
        // stored (each output row depends only on its own A row).
        const int valid_rows = min(kBM, s_offsets[e] + __ldg(args.counts + e) - mt * kBM);
        const uint32_t a_bytes = static_cast<uint32_t>((valid_rows + 15) / 16) * 16 * kRowBytesPerStage;
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
            fail_bits |= MOE_DEVICE_TIMEOUT_PRODUCER;
            break;
          }
          const int kb_here = min(4, (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK);
          const uint32_t sf_bytes = !Tr::kScaled ? 0u : ((FMT == MOE_NVFP4) ? 512u * kb_here : 512u);
          uint8_t* st = smem + stage * Tr::kStageBytes;
          mbar_arrive_expect_tx(&full_bar[stage], a_bytes + Tr::kBBytes + sf_bytes * (1 + kBN / 128));
          bulk_load(st, a_tiles + static_cast<int64_t>(kt) * Tr::kABytes, a_bytes, &full_bar[stage], pol_a);
          bulk_load(st + Tr::kABytes, b_tiles + static_cast<int64_t>(kt) * Tr::kBBytes, Tr::kBBytes, &full_bar[stage],
                    pol_w);
          if (Tr::kScaled) {
            bulk_load(st + Tr::kSfaOff, a_sf + kt * Tr::kSfBytes128, sf_bytes, &full_bar[stage], pol_a);
#pragma unroll
            for (int h = 0; h < kBN / 128; ++h)
              bulk_load(st + Tr::kSfbOff + h * Tr::kSfBytes128, b_sf + h * args.sf_rb_stride + kt * Tr::kSfBytes128,
                        sf_bytes, &full_bar[stage], pol_w);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t d_tmem = tmem_base;
      // Descriptors of stage 0; a stage adds kStageDesc 16-byte units (the
      // 14-bit start field never carries: shared memory is below 256 KB).
      const uint64_t adesc0 = make_desc_sw128(smem_u32(smem));
      const uint64_t bdesc0 = make_desc_sw128(smem_u32(smem) + Tr::kABytes);
      constexpr uint32_t kStageDesc = Tr::kStageBytes >> 4;
      const int full_stages = args.K / Tr::kElemsPerStage;  // stages with all 4 k blocks
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar, acc_phase ^ 1u, abort_flag)) {
          fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt) {
          // the scale copiers have seen the stage's operands land and issued
          // their copies (the operand wait then returns at once)
          if ((Tr::kScaled && !mbar_wait(&sf_bar[stage], phase, abort_flag)) ||
              !mbar_wait(&full_bar[stage], phase, abort_flag)) {
            fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
            ok = false;
            break;
          }
          tc_fence_after();
          // The issuing thread's own instruction latency is on the tensor
          // pipe's critical path: whole stages issue their four MMAs
          // unrolled, with operands computed independently of each other.
          const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage) * kStageDesc;
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(stage) * kStageDesc;
          const uint32_t sfa = tmem_base + Tr::kTmemSfa + stage * kSfColsPerStage<FMT>;
          const uint32_t sfb = sfa + Tr::kSfaCols;
          const uint32_t acc0 = kt != 0 ? 1u : 0u;
          if (kt < full_stages) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint32_t accum = kb != 0 ? 1u : acc0;
              if (FMT == MOE_BF16) {
                tc_mma_bf16(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_bf16(kBN), accum);
              } else if (FMT == MOE_NVFP4) {
                tc_mma_nvfp4(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_nvfp4(kBN), sfa + 4 * kb,
                             sfb + (kBN / 32) * kb, accum);
              } else {
                const uint32_t sel = static_cast<uint32_t>(kb) << 30;
                tc_mma_mxfp8(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_mxfp8(kBN, kb), sfa | sel, sfb | sel,
                             accum);
              }
            }
          } else {
            const int kb_here = (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK;
            for (int kb = 0; kb < kb_here; ++kb) {
              const uint32_t accum = kb != 0 ? 1u : acc0;
              if (FMT == MOE_BF16) {
                tc_mma_bf16(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_bf16(kBN), accum);
              } else if (FMT == MOE_NVFP4) {
                tc_mma_nvfp4(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_nvfp4(kBN), sfa + 4 * kb,
                             sfb + (kBN / 32) * kb, accum);
              } else {
                const uint32_t sel = static_cast<uint32_t>(kb) << 30;
                tc_mma_mxfp8(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc_mxfp8(kBN, kb), sfa | sel, sfb | sel,
                             accum);
              }
            }
          }
          tc_commit(&empty_bar[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar);
        acc_phase ^= 1u;
      }
    }
  } else if (warp >= kThreads / 32) {
    // ------------------------------------------------------------ scale copiers
    const int part = warp - kThreads / 32;  // copies the scales of k blocks part, part + kCopierWarps, ...
    if (lane == 0 && Tr::kScaled) {
      int stage = 0;
      uint32_t phase = 0;
      // scale-atom descriptor of stage 0's A scales; every other atom is a
      // constant number of 16-byte units away
      const uint64_t sdesc0 = make_desc_sf(smem_u32(smem) + Tr::kSfaOff);
      constexpr uint32_t kStageDesc = Tr::kStageBytes >> 4;
      const int full_stages = args.K / Tr::kElemsPerStage;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt) {
          // The stage's TMEM scale columns were last read by the MMAs of the
          // same stage one ring turn ago; those completed before the stage
          // was released and refilled, i.e. before this wait returns.
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
            fail_bits |= MOE_DEVICE_TIMEOUT_MMA;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t sdesc = sdesc0 + static_cast<uint64_t>(stage) * kStageDesc;  // this stage's A atom 0
          constexpr uint32_t kSfbDesc = (Tr::kSfbOff - Tr::kSfaOff) >> 4;
          constexpr uint32_t kAtomDesc = 512 >> 4;
          const uint32_t sfa = tmem_base + Tr::kTmemSfa + stage * kSfColsPerStage<FMT>;
          const uint32_t sfb = sfa + Tr::kSfaCols;
          if (FMT == MOE_NVFP4) {
            // this warp's k blocks part, part + kCopierWarps, ...
            const int kb_here = kt < full_stages ? 4 : (args.K - kt * Tr::kElemsPerStage) / Tr::kMmaK;
            for (int kb = part; kb < kb_here; kb += kCopierWarps) {
              tc_cp_sf_atom(sfa + 4 * kb, sdesc + kAtomDesc * kb);
#pragma unroll
              for (int h = 0; h < kBN / 128; ++h)
                tc_cp_sf_atom(sfb + (kBN / 32) * kb + 4 * h,
                              sdesc + kSfbDesc + h * (Tr::kSfBytes128 >> 4) + kAtomDesc * kb);
            }
          } else if (part == 0) {
            tc_cp_sf_atom(sfa, sdesc);
            tc_cp_sf_atom(sfb, sdesc + kSfbDesc);
          } else {
#pragma unroll
            for (int h = 1; h < kBN / 128; ++h) tc_cp_sf_atom(sfb + 4 * h, sdesc + kSfbDesc + h * (Tr::kSfBytes128 >> 4));
          }
          // Signal that the copies are issued, not that they are complete:
          // tcgen05.cp -> tcgen05.mma is a pipelined pair, so the MMA
          // thread's fence::after_thread_sync after this barrier orders its
          // MMAs behind these copies in the tensor pipe.
          tc_fence_before();
          mbar_arrive(&sf_bar[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warps 2..9: quarter q = warp % 4 of the TMEM lanes (rows), half of the
    // accumulator columns.  Each thread copies its 128 columns to registers,
    // hands the accumulator back to the MMA warp at once, and then does the
    // epilogue math while the next tile's MMAs run.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_l = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + half * (kBN / 2);
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, s_offsets, E, n_tiles, args.expert_map, args.n_weights);
      const int mt = tc.mt, nt = tc.nt, e = tc.e;
      const int valid_rows = s_offsets[e] + __ldg(args.counts + e) - mt * kBM;
      if (tc.bad && warp == 2 && lane == 0) fail_bits |= MOE_DEVICE_BAD_GROUP_EXPERT;
      const bool valid = row_l < valid_rows;
      const int64_t row = static_cast<int64_t>(mt) * kBM + row_l;
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
      mbar_arrive(tempty_bar);
      acc_phase ^= 1u;
      if (!valid) continue;
      epilogue_rows<FMT, GATEUP>(args, acc, row, tc.we, nt, half);
    }
  }

  if (fail_bits != 0u && args.status != nullptr) atomicOr(args.status, fail_bits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every role has left its loop; the abort flag no longer changes.  After a
  // normal run nothing is in flight (each stage's copies landed before its
  // MMAs ran, each scale copy finished before its MMAs ran, the last MMAs
  // before the epilogue's last wait).  After an abort, wait for what is.
  if (*abort_flag) {
    bool drained = true;
    if (warp == 0 && lane == 0) {
      // a stage's copies complete its full barrier phase whether or not the
      // MMA warp consumed it, and a stage is re-armed only after it is freed
      for (int st = 0; st < kStages; ++st)
        if ((armed >> st) & 1u) drained = mbar_wait_drain(&full_bar[st], (armed_par >> st) & 1u) && drained;
    } else if ((warp == 1 || warp >= kThreads / 32) && lane == 0) {
      // MMAs and scale copies this thread issued: one arrival each on the
      // drain barrier once they have completed
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

// ---------------------------------------------------------------- host side

template <int FMT, bool GATEUP>
static cudaError_t launch_one(const GemmArgs& a, cudaStream_t stream) {
  using Tr = GemmTraits<FMT, kBN, kStages>;
  const size_t smem = 1024 + kStages * Tr::kStageBytes + (3 * kStages + 3) * 8 + 16 + (a.E + 1) * 4;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  // per device: the kernel's shared-memory limit is raised once and the SM
  // count read once (host threads may launch concurrently; both are idempotent)
  static std::atomic<int> sm_count[64];
  int sms = (dev < 64) ? sm_count[dev].load(std::memory_order_relaxed) : 0;
  if (sms == 0) {
    // the largest size any supported E needs (E <= 1024)
    const size_t smem_max = 1024 + kStages * Tr::kStageBytes + (3 * kStages + 3) * 8 + 16 + 1025 * 4;
    err = cudaFuncSetAttribute(moe_gemm_kernel<FMT, GATEUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_max));
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    if (dev < 64) sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  return launch_pdl(moe_gemm_kernel<FMT, GATEUP>, dim3(sms), dim3(kThreadsOne), smem, stream, a);
}

size_t gemm_smem_bytes(int fmt, int E) {
  const int sb = (fmt == MOE_NVFP4) ? GemmTraits<MOE_NVFP4, kBN, kStages>::kStageBytes
                 : (fmt == MOE_MXFP8) ? GemmTraits<MOE_MXFP8, kBN, kStages>::kStageBytes
                                      : GemmTraits<MOE_BF16, kBN, kStages>::kStageBytes;
  return 1024 + kStages * sb + (3 * kStages + 3) * 8 + 16 + (E + 1) * 4;
}

cudaError_t launch_gemm_pair(const GemmLaunch& g, const GemmArgs& a, cudaStream_t stream);  // gemm_pair.cu

namespace {
// Which kernel serves block-scaled GEMMs: one SM per tile unless
// MOE_B200_GEMM = "pair" asks for the SM-pair kernel (kept as an option: it
// is exact but measured slower than one SM per tile at prefill).
int gemm_mode() {
  static const int mode = [] {
    const char* v = std::getenv("MOE_B200_GEMM");
    if (v == nullptr) return 0;
    return std::strcmp(v, "pair") == 0 ? 2 : 1;
  }();
  return mode;
}
}  // namespace

cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t stream) {
  const int bits = (g.fmt == MOE_NVFP4) ? 4 : (g.fmt == MOE_MXFP8 ? 8 : 16);
  const int sfvec = (g.fmt == MOE_MXFP8) ? 32 : 16;
  GemmArgs a;
  a.a_codes = g.a_codes;
  a.b_codes = g.b_codes;
  a.kb = kb_padded(g.K, bits);
  a.b_expert_stride = static_cast<int64_t>(g.n_rows_b) * a.kb;
  // BF16: h carries the adapter K tile after its d_ffn channels
  a.h_kb = g.gateup ? kb_padded(g.n_rows_b / 2 + (g.fmt == MOE_BF16 ? 64 : 0), bits) : 0;
  a.a_sf = g.a_sf;
  a.b_sf = g.b_sf;
  a.offsets = g.offsets;
  a.counts = g.counts;
  a.a_scale = g.a_scale;
  a.w_scales = g.w_scales;
  a.h_scale = g.h_scale;
  a.h_codes = g.h_codes;
  a.h_sf = g.h_sf;
  a.dbg = g.dbg;
  a.out = static_cast<__nv_bfloat16*>(g.out);
  a.status = g.status;
  a.expert_map = g.expert_map;
  a.n_weights = g.expert_map != nullptr ? g.n_weights : g.E;
  a.E = g.E;
  a.K = g.K;
  a.n_rows_b = g.n_rows_b;
  a.sf_rb_stride = static_cast<int64_t>(g.K / sfvec) * 128;
  a.b_sf_expert_stride = static_cast<int64_t>(g.n_rows_b) * (g.K / sfvec);
  if (g.fmt != MOE_BF16 && g.R_max > 0) {
    if (gemm_mode() == 2) return launch_gemm_pair(g, a, stream);
  }
  if (g.fmt == MOE_NVFP4)
    return g.gateup ? launch_one<MOE_NVFP4, true>(a, stream) : launch_one<MOE_NVFP4, false>(a, stream);
  if (g.fmt == MOE_BF16)
    return g.gateup ? launch_one<MOE_BF16, true>(a, stream) : launch_one<MOE_BF16, false>(a, stream);
  return g.gateup ? launch_one<MOE_MXFP8, true>(a, stream) : launch_one<MOE_MXFP8, false>(a, stream);
}

}  // namespace moe
