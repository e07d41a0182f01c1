// C ABI of the routed MoE expert layer: argument validation, sizes, layout
// queries, and dispatch to the kernels.  See include/moe_b200.h for the
// contract of every entry point.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr int64_t kMaxTokens = int64_t(1) << 20;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A block-scale buffer argument: unused (may be NULL) for BF16, required and
// aligned for the block-scaled formats.
bool sf_ok(const moe_config* cfg, const void* sf) {
  return cfg->fmt == MOE_BF16 ? (sf == nullptr || aligned16(sf)) : (sf != nullptr && aligned16(sf));
}

int bits_of(const moe_config* c) { return c->fmt == MOE_NVFP4 ? 4 : (c->fmt == MOE_MXFP8 ? 8 : 16); }
int sfvec_of(const moe_config* c) { return c->fmt == MOE_MXFP8 ? 32 : 16; }
// bytes of one tiled operand row of K elements (BF16: plus the adapter K tile)
int64_t row_bytes(const moe_config* c, int64_t K) {
  return c->fmt == MOE_BF16 ? 2 * K + 128 : moe::kb_padded(K, bits_of(c));
}

moe_status check(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->fmt != MOE_NVFP4 && c->fmt != MOE_MXFP8 && c->fmt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->num_experts < 1 || c->num_experts > 1024) return MOE_ERR_UNSUPPORTED;
  if (c->top_k < 1 || c->top_k > 8 || c->top_k > c->num_experts) return MOE_ERR_UNSUPPORTED;
  if (c->d_model < 256 || c->d_model % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->d_ffn < 128 || c->d_ffn % 128 != 0) return MOE_ERR_UNSUPPORTED;
  // row indices of all experts' weights stay within int32
  if (static_cast<int64_t>(c->num_experts) * 2 * c->d_ffn >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(c->num_experts) * c->d_model >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_T(int64_t T) { return (T < 0 || T > kMaxTokens) ? MOE_ERR_UNSUPPORTED : MOE_OK; }

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int64_t max_rows(const moe_config* c, int64_t T) {
  const int64_t slots = T * c->top_k;
  const int64_t touched = slots < c->num_experts ? slots : c->num_experts;
  const int64_t r = slots + 127 * touched;
  return (r + 127) / 128 * 128;
}

void layout(const moe_config* c, moe_weights_layout* L) {
  const int64_t E = c->num_experts, H = c->d_model, I = c->d_ffn;
  const int b = bits_of(c), v = sfvec_of(c);
  auto up256 = [](int64_t x) { return (x + 255) / 256 * 256; };
  int64_t off = 0;
  const bool bf16 = c->fmt == MOE_BF16;
  (void)b;
  L->w13_codes = off;
  off = up256(off + E * 2 * I * row_bytes(c, H));
  L->w13_sf = off;  // BF16: the adapters' A of gate and up, 64 rows per expert
  off = up256(off + (bf16 ? E * 64 * 2 * H : E * 2 * I * H / v));
  L->w2_codes = off;
  off = up256(off + E * H * row_bytes(c, I));
  L->w2_sf = off;   // BF16: A of down and 32 zero rows
  off = up256(off + (bf16 ? E * 64 * 2 * I : E * H * I / v));
  L->scales = off;
  off = up256(off + E * 3 * 4);
  L->total_bytes = off;
}

}  // namespace

extern "C" {

moe_status moe_check_config(const moe_config* cfg) { return check(cfg); }

moe_status moe_get_weights_layout(const moe_config* cfg, moe_weights_layout* out) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  layout(cfg, out);
  return MOE_OK;
}

int64_t moe_max_rows(const moe_config* cfg, int64_t T) {
  if (check(cfg) != MOE_OK || check_T(T) != MOE_OK) return -1;
  return max_rows(cfg, T);
}

int64_t moe_codes_bytes(const moe_config* cfg, int64_t rows, int64_t K) {
  if (check(cfg) != MOE_OK || rows < 0 || K <= 0 || rows % 128 != 0) return -1;
  if (cfg->fmt == MOE_BF16 && K % 64 != 0) return -1;
  return rows * row_bytes(cfg, K);
}

int64_t moe_sf_bytes(const moe_config* cfg, int64_t rows, int64_t K) {
  if (check(cfg) != MOE_OK || rows < 0 || K <= 0 || rows % 128 != 0) return -1;
  if (cfg->fmt == MOE_BF16) return 0;  // no block scales
  if (K % (4 * sfvec_of(cfg)) != 0) return -1;
  return rows * K / sfvec_of(cfg);
}

int64_t moe_sf_offset(int64_t row, int64_t col, int64_t nsf) { return moe::sf_offset(row, col, nsf); }

int64_t moe_route_workspace_bytes(const moe_config* cfg, int64_t T) {
  if (check(cfg) != MOE_OK || check_T(T) != MOE_OK) return -1;
  return moe::route_workspace_bytes(cfg->num_experts, T);
}

moe_status moe_pack_weights_bf16(const moe_config* cfg, int32_t expert_begin, int32_t expert_count,
                                 const void* w_gate, const void* w_up, const void* w_down, const void* lora_a_gate,
                                 const void* lora_b_gate, const void* lora_a_up, const void* lora_b_up,
                                 const void* lora_a_down, const void* lora_b_down, int32_t lora_rank,
                                 float lora_scaling, void* packed, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if (cfg->fmt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (expert_begin < 0 || expert_count < 0 || expert_begin + expert_count > cfg->num_experts)
    return MOE_ERR_INVALID_ARG;
  if (expert_count == 0) return MOE_OK;
  if (!w_gate || !w_up || !w_down || !packed) return MOE_ERR_INVALID_ARG;
  const void* lora[6] = {lora_a_gate, lora_b_gate, lora_a_up, lora_b_up, lora_a_down, lora_b_down};
  int given = 0;
  for (const void* p : lora) given += p != nullptr;
  if (given != 0 && given != 6) return MOE_ERR_INVALID_ARG;  // all six adapter matrices, or none
  if (given == 6 && (lora_rank < 1 || lora_rank > 32)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(packed)) return MOE_ERR_INVALID_ARG;
  if (given == 6 && (!aligned16(lora_a_gate) || !aligned16(lora_a_up) || !aligned16(lora_a_down)))
    return MOE_ERR_INVALID_ARG;
  moe_weights_layout L;
  layout(cfg, &L);
  uint8_t* base = static_cast<uint8_t*>(packed);
  return from_cuda(moe::launch_pack_bf16(
      cfg->d_model, cfg->d_ffn, expert_begin, expert_count, w_gate, w_up, w_down, lora_a_gate, lora_a_up,
      lora_a_down, lora_b_gate, lora_b_up, lora_b_down, given == 6 ? lora_rank : 0, lora_scaling, base + L.w13_codes,
      base + L.w13_sf, base + L.w2_codes, base + L.w2_sf, reinterpret_cast<float*>(base + L.scales),
      static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_weights(const moe_config* cfg, int32_t expert_begin, int32_t expert_count,
                                const float* w_gate, const float* w_up, const float* w_down, void* packed,
                                void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if (cfg->fmt == MOE_BF16) return MOE_ERR_UNSUPPORTED;  // moe_pack_weights_bf16
  if (expert_begin < 0 || expert_count < 0 || expert_begin + expert_count > cfg->num_experts)
    return MOE_ERR_INVALID_ARG;
  if (expert_count == 0) return MOE_OK;
  if (!w_gate || !w_up || !w_down || !packed) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(packed)) return MOE_ERR_INVALID_ARG;
  moe_weights_layout L;
  layout(cfg, &L);
  uint8_t* base = static_cast<uint8_t*>(packed);
  return from_cuda(moe::launch_quantize_weights(
      cfg->fmt, cfg->num_experts, cfg->d_model, cfg->d_ffn, expert_begin, expert_count, w_gate, w_up, w_down,
      base + L.w13_codes, base + L.w13_sf, base + L.w2_codes, base + L.w2_sf,
      reinterpret_cast<float*>(base + L.scales), static_cast<cudaStream_t>(stream)));
}

moe_status moe_route_topk(const moe_config* cfg, int64_t T, const float* logits, int32_t* topk_ids,
                          float* topk_w, int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                          int32_t* slot_to_row, void* workspace, int64_t workspace_bytes, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  // sorted_slots has max_rows(T) rows: none for an empty batch
  if (!expert_counts || !expert_offsets || (T > 0 && !sorted_slots)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_ids || !topk_w || !slot_to_row || !workspace)) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe::route_workspace_bytes(cfg->num_experts, T)) return MOE_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_route(logits, static_cast<int>(T), cfg->num_experts, cfg->top_k, topk_ids, topk_w,
                                     expert_counts, expert_offsets, sorted_slots, slot_to_row, max_rows(cfg, T),
                                     workspace, static_cast<cudaStream_t>(stream)));
}

moe_status moe_router_topk(const moe_config* cfg, int64_t T, const void* x_bf16, const void* w_router_bf16,
                           float* logits_out, int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                           int32_t* expert_offsets, int32_t* sorted_slots, int32_t* slot_to_row, void* workspace,
                           int64_t workspace_bytes, uint32_t* status_word, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  if (cfg->num_experts > 512) return MOE_ERR_UNSUPPORTED;  // all scores of a token in one TMEM accumulator
  if (!expert_counts || !expert_offsets || (T > 0 && !sorted_slots)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x_bf16 || !w_router_bf16 || !topk_ids || !topk_w || !slot_to_row || !workspace))
    return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe::route_workspace_bytes(cfg->num_experts, T)) return MOE_ERR_WORKSPACE;
  if ((x_bf16 && !aligned16(x_bf16)) || (w_router_bf16 && !aligned16(w_router_bf16)) ||
      (workspace && !aligned16(workspace)) || (logits_out && !aligned16(logits_out)))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = cfg->num_experts, k = cfg->top_k;
  cudaError_t err = moe::route_prepare(static_cast<int>(T), E, expert_counts, expert_offsets, sorted_slots,
                                       max_rows(cfg, T), workspace, st);
  if (err != cudaSuccess || T == 0) return from_cuda(err);
  err = moe::launch_router_topk(x_bf16, w_router_bf16, logits_out, static_cast<int>(T), E, cfg->d_model, k, topk_ids,
                                topk_w, workspace, status_word, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return from_cuda(moe::route_finish(static_cast<int>(T), E, k, topk_ids, expert_counts, expert_offsets, sorted_slots,
                                     slot_to_row, max_rows(cfg, T), workspace, st));
}

moe_status moe_permute(const moe_config* cfg, int64_t T, const void* x_bf16, const float* act_scale,
                       const int32_t* slot_to_row, void* a_codes, void* a_sf, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !slot_to_row || !a_codes) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && !act_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(a_codes) || !sf_ok(cfg, a_sf)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute(cfg->fmt, static_cast<int>(T), cfg->d_model, cfg->top_k, x_bf16, act_scale,
                                       slot_to_row, static_cast<uint8_t*>(a_codes), static_cast<uint8_t*>(a_sf),
                                       static_cast<cudaStream_t>(stream)));
}

static moe_status gemm_common(const moe_config* cfg, int64_t T, const void* packed, const int32_t* expert_offsets,
                              const int32_t* expert_counts) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  if (!packed || !expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
  if (!aligned16(packed)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Row groups of the expert GEMMs: experts (group_expert null) or segments
// naming the expert whose weights they use.
struct Groups {
  int n;
  const int32_t* offsets;
  const int32_t* counts;
  const int32_t* expert;
  int64_t R_max;  // rows the buffers hold (bounds the adapter shrink's grid and the tensor maps)
  int64_t slots;  // T * k when known (selects the GEMM kernel), else 0
};

// gate/up GEMM + SwiGLU + h in the layer format.  BF16: the adapter shrink
// of A first (into A's adapter K tile), the GEMM over d_model + 64, then the
// shrink of h (into h's adapter K tile) for the down GEMM.
static moe_status run_gateup(const moe_config* cfg, const Groups& G, const uint8_t* base, const void* a_codes,
                             const void* a_sf, const float* act_scale, const float* inter_scale, void* h_codes,
                             void* h_sf, float* dbg, uint32_t* status, cudaStream_t st) {
  moe_weights_layout L;
  layout(cfg, &L);
  const bool bf16 = cfg->fmt == MOE_BF16;
  const float* scales = reinterpret_cast<const float*>(base + L.scales);
  if (bf16) {
    const cudaError_t err = moe::launch_lora_shrink(
        static_cast<uint8_t*>(const_cast<void*>(a_codes)), 2 * int64_t(cfg->d_model) + 128, cfg->d_model,
        base + L.w13_sf, scales, G.offsets, G.counts, G.expert, cfg->num_experts, G.n, G.R_max, status, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  moe::GemmLaunch g{};
  g.fmt = cfg->fmt;
  g.gateup = true;
  g.E = G.n;
  g.R_max = G.R_max;
  g.slots = G.slots;
  g.K = cfg->d_model + (bf16 ? 64 : 0);
  g.n_rows_b = 2 * cfg->d_ffn;
  g.a_codes = static_cast<const uint8_t*>(a_codes);
  g.a_sf = static_cast<const uint8_t*>(a_sf);
  g.b_codes = base + L.w13_codes;
  g.b_sf = base + L.w13_sf;
  g.offsets = G.offsets;
  g.counts = G.counts;
  g.expert_map = G.expert;
  g.n_weights = cfg->num_experts;
  g.a_scale = act_scale;
  g.w_scales = scales;
  g.h_scale = inter_scale;
  g.h_codes = static_cast<uint8_t*>(h_codes);
  g.h_sf = static_cast<uint8_t*>(h_sf);
  g.dbg = dbg;
  g.status = status;
  if (moe::launch_gemm(g, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (bf16) {
    return from_cuda(moe::launch_lora_shrink(static_cast<uint8_t*>(h_codes), 2 * int64_t(cfg->d_ffn) + 128,
                                             cfg->d_ffn, base + L.w2_sf, scales, G.offsets, G.counts, G.expert,
                                             cfg->num_experts, G.n, G.R_max, status, st));
  }
  return MOE_OK;
}

// down GEMM -> bf16 rows (BF16: over d_ffn + 64, the adapter tile of h).
static moe_status run_down(const moe_config* cfg, const Groups& G, const uint8_t* base, const void* h_codes,
                           const void* h_sf, const float* inter_scale, void* down_out, uint32_t* status,
                           cudaStream_t st) {
  moe_weights_layout L;
  layout(cfg, &L);
  moe::GemmLaunch g{};
  g.fmt = cfg->fmt;
  g.gateup = false;
  g.E = G.n;
  g.R_max = G.R_max;
  g.slots = G.slots;
  g.K = cfg->d_ffn + (cfg->fmt == MOE_BF16 ? 64 : 0);
  g.n_rows_b = cfg->d_model;
  g.a_codes = static_cast<const uint8_t*>(h_codes);
  g.a_sf = static_cast<const uint8_t*>(h_sf);
  g.b_codes = base + L.w2_codes;
  g.b_sf = base + L.w2_sf;
  g.offsets = G.offsets;
  g.counts = G.counts;
  g.expert_map = G.expert;
  g.n_weights = cfg->num_experts;
  g.a_scale = inter_scale;
  g.w_scales = reinterpret_cast<const float*>(base + L.scales);
  g.out = down_out;
  g.status = status;
  return from_cuda(moe::launch_gemm(g, st));
}

moe_status moe_forward_gateup(const moe_config* cfg, int64_t T, const void* packed, const void* a_codes,
                              const void* a_sf, const float* act_scale, const float* inter_scale,
                              const int32_t* expert_offsets, const int32_t* expert_counts, void* h_codes,
                              void* h_sf, float* gateup_debug, uint32_t* status_word, void* stream) {
  moe_status s = gemm_common(cfg, T, packed, expert_offsets, expert_counts);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!a_codes || !h_codes || !aligned16(a_codes) || !aligned16(h_codes)) return MOE_ERR_INVALID_ARG;
  if (!sf_ok(cfg, a_sf) || !sf_ok(cfg, h_sf)) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && (!act_scale || !inter_scale)) return MOE_ERR_INVALID_ARG;
  if (gateup_debug && !aligned16(gateup_debug)) return MOE_ERR_INVALID_ARG;
  const Groups G{cfg->num_experts, expert_offsets, expert_counts, nullptr, max_rows(cfg, T), T * cfg->top_k};
  return run_gateup(cfg, G, static_cast<const uint8_t*>(packed), a_codes, a_sf, act_scale, inter_scale, h_codes,
                    h_sf, gateup_debug, status_word, static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_down(const moe_config* cfg, int64_t T, const void* packed, const void* h_codes,
                            const void* h_sf, const float* inter_scale, const int32_t* expert_offsets,
                            const int32_t* expert_counts, void* down_out, uint32_t* status_word, void* stream) {
  moe_status s = gemm_common(cfg, T, packed, expert_offsets, expert_counts);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!h_codes || !down_out || !aligned16(h_codes) || !aligned16(down_out)) return MOE_ERR_INVALID_ARG;
  if (!sf_ok(cfg, h_sf)) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && !inter_scale) return MOE_ERR_INVALID_ARG;
  const Groups G{cfg->num_experts, expert_offsets, expert_counts, nullptr, max_rows(cfg, T), T * cfg->top_k};
  return run_down(cfg, G, static_cast<const uint8_t*>(packed), h_codes, h_sf, inter_scale, down_out, status_word,
                  static_cast<cudaStream_t>(stream));
}

moe_status moe_forward(const moe_config* cfg, int64_t T, const void* packed, const void* a_codes,
                       const void* a_sf, const float* act_scale, const float* inter_scale,
                       const int32_t* expert_offsets, const int32_t* expert_counts, void* h_codes, void* h_sf,
                       void* down_out, float* gateup_debug, uint32_t* status_word, void* stream) {
  moe_status s = moe_forward_gateup(cfg, T, packed, a_codes, a_sf, act_scale, inter_scale, expert_offsets,
                                    expert_counts, h_codes, h_sf, gateup_debug, status_word, stream);
  if (s != MOE_OK) return s;
  return moe_forward_down(cfg, T, packed, h_codes, h_sf, inter_scale, expert_offsets, expert_counts, down_out,
                          status_word, stream);
}

moe_status moe_forward_grouped(const moe_config* cfg, int32_t num_groups, int64_t max_rows_, const void* packed,
                               const void* a_codes, const void* a_sf, const float* act_scale,
                               const float* inter_scale, const int32_t* group_offsets, const int32_t* group_counts,
                               const int32_t* group_expert, void* h_codes, void* h_sf, void* down_out,
                               float* gateup_debug, uint32_t* status_word, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if (num_groups < 0 || num_groups > 1024) return MOE_ERR_UNSUPPORTED;
  if (max_rows_ < 0 || max_rows_ % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (num_groups == 0 || max_rows_ == 0) return MOE_OK;
  if (!packed || !a_codes || !group_offsets || !group_counts || !group_expert || !h_codes || !down_out)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(a_codes) || !aligned16(h_codes) || !aligned16(down_out) ||
      (gateup_debug && !aligned16(gateup_debug)) || !sf_ok(cfg, a_sf) || !sf_ok(cfg, h_sf))
    return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && (!act_scale || !inter_scale)) return MOE_ERR_INVALID_ARG;
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Groups G{num_groups, group_offsets, group_counts, group_expert, max_rows_, 0};
  s = run_gateup(cfg, G, base, a_codes, a_sf, act_scale, inter_scale, h_codes, h_sf, gateup_debug, status_word, st);
  if (s != MOE_OK) return s;
  return run_down(cfg, G, base, h_codes, h_sf, inter_scale, down_out, status_word, st);
}

moe_status moe_unpermute_combine(const moe_config* cfg, int64_t T, const void* down_out, const float* topk_w,
                                 const int32_t* slot_to_row, void* y_bf16, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!down_out || !topk_w || !slot_to_row || !y_bf16) return MOE_ERR_INVALID_ARG;
  if (!aligned16(down_out) || !aligned16(y_bf16)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine(static_cast<int>(T), cfg->d_model, cfg->top_k, down_out, topk_w, slot_to_row,
                                       y_bf16, static_cast<cudaStream_t>(stream)));
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null, misaligned or out-of-range)";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration or size";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

}  // extern "C"
