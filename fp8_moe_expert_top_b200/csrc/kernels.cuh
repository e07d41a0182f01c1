// Host-side launchers of the library's kernels (internal).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

int64_t route_workspace_bytes(int E, int64_t T);
cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                         int32_t* slot_to_row, int64_t R_max, void* workspace, cudaStream_t stream);

// The routing steps around the top-k: zero the token bitmaps and mark every
// row of sorted_slots as padding (prepare), then per-expert counts, padded
// offsets and the slot scatter from the bitmaps (finish).  Small batches
// (route_small) need no prepare step and no bitmaps from the top-k: the
// finish step builds them itself from topk_ids in one CTA.
constexpr int kSmallWords = 8192;  // E * ceil(T / 32) bitmap words of a small batch
bool route_small(int T, int E);
cudaError_t route_prepare(int T, int E, int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                          int64_t R_max, void* workspace, cudaStream_t stream);
cudaError_t route_finish(int T, int E, int k, const int32_t* topk_ids, int32_t* expert_counts,
                         int32_t* expert_offsets, int32_t* sorted_slots, int32_t* slot_to_row, int64_t R_max,
                         void* workspace, cudaStream_t stream);

// Router scores fused with the top-k (logits = x W_r^T on tcgen05, then the
// same top-k, softmax and bitmaps as route_topk_kernel); E <= 512.
cudaError_t launch_router_topk(const void* x, const void* w_router, float* logits_out, int T, int E, int H, int k,
                               int32_t* topk_ids, float* topk_w, void* workspace, uint32_t* status,
                               cudaStream_t stream);

cudaError_t launch_permute(int fmt, int T, int H, int k, const void* x, const float* act_scale,
                           const int32_t* slot_to_row, uint8_t* a_codes, uint8_t* a_sf, cudaStream_t stream);

cudaError_t launch_combine(int T, int H, int k, const void* down_out, const float* topk_w,
                           const int32_t* slot_to_row, void* y, cudaStream_t stream);

cudaError_t launch_quantize_weights(int fmt, int E, int H, int I, int expert_begin, int expert_count,
                                    const float* w_gate, const float* w_up, const float* w_down, uint8_t* w13_codes,
                                    uint8_t* w13_sf, uint8_t* w2_codes, uint8_t* w2_sf, float* scales,
                                    cudaStream_t stream);

// BF16 experts: bf16 weights and adapters into the tiled layout (see the
// header's MOE_BF16 layout), and the adapter shrink z = s_e (a A_e^T) of the
// rows of a tiled bf16 operand (kb bytes per row, K elements plus the adapter
// tile), written into that tile.
cudaError_t launch_pack_bf16(int H, int I, int expert_begin, int expert_count, const void* w_gate, const void* w_up,
                             const void* w_down, const void* a_gate, const void* a_up, const void* a_down,
                             const void* b_gate, const void* b_up, const void* b_down, int rank, float scaling,
                             uint8_t* w13, uint8_t* s13, uint8_t* w2, uint8_t* s2, float* scales,
                             cudaStream_t stream);
cudaError_t launch_lora_shrink(uint8_t* a, int64_t kb, int K, const uint8_t* w, const float* scales,
                               const int32_t* offsets, const int32_t* counts, const int32_t* expert_map,
                               int n_weights, int E, int64_t R_max, uint32_t* status, cudaStream_t stream);

struct GemmLaunch {
  int fmt;
  bool gateup;
  int E, K, n_rows_b;     // K in elements, rows of B per expert (2I or H)
  int64_t R_max;
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const uint8_t* b_codes;
  const uint8_t* b_sf;
  const int32_t* offsets;
  const int32_t* counts;
  const float* a_scale;   // device scalar or null (MXFP8)
  const float* w_scales;  // [E][3]
  const float* h_scale;   // gate/up: tensor scale of h (NVFP4) or null
  uint8_t* h_codes;
  uint8_t* h_sf;
  float* dbg;
  void* out;              // down: bf16 [R_max][H]
  uint32_t* status;
  const int32_t* expert_map;  // optional [E]: row group -> expert of the packed weights
  int n_weights;              // experts in the packed weights (with expert_map)
  int64_t slots;              // token slots routed (T * k), 0 when unknown; selects the SM-pair kernel
};
cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t stream);

}  // namespace moe
