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

int bits_of(const moe_config* c) { return c->fmt == MOE_NVFP4 ? 4 : 8; }
int sfvec_of(const moe_config* c) { return c->fmt == MOE_NVFP4 ? 16 : 32; }

moe_status check(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->fmt != MOE_NVFP4 && c->fmt != MOE_MXFP8) return MOE_ERR_UNSUPPORTED;
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
  L->w13_codes = off;
  off = up256(off + E * 2 * I * moe::kb_padded(H, b));
  L->w13_sf = off;
  off = up256(off + E * 2 * I * H / v);
  L->w2_codes = off;
  off = up256(off + E * H * moe::kb_padded(I, b));
  L->w2_sf = off;
  off = up256(off + E * H * I / v);
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
  return rows * moe::kb_padded(K, bits_of(cfg));
}

int64_t moe_sf_bytes(const moe_config* cfg, int64_t rows, int64_t K) {
  if (check(cfg) != MOE_OK || rows < 0 || K <= 0 || rows % 128 != 0 || K % (4 * sfvec_of(cfg)) != 0) return -1;
  return rows * K / sfvec_of(cfg);
}

int64_t moe_sf_offset(int64_t row, int64_t col, int64_t nsf) { return moe::sf_offset(row, col, nsf); }

int64_t moe_route_workspace_bytes(const moe_config* cfg, int64_t T) {
  if (check(cfg) != MOE_OK || check_T(T) != MOE_OK) return -1;
  return moe::route_workspace_bytes(cfg->num_experts, T);
}

moe_status moe_quantize_weights(const moe_config* cfg, int32_t expert_begin, int32_t expert_count,
                                const float* w_gate, const float* w_up, const float* w_down, void* packed,
                                void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
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
  if (!expert_counts || !expert_offsets || !sorted_slots) return MOE_ERR_INVALID_ARG;
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
  if (!expert_counts || !expert_offsets || !sorted_slots) return MOE_ERR_INVALID_ARG;
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
                                     slot_to_row, workspace, st));
}

moe_status moe_permute(const moe_config* cfg, int64_t T, const void* x_bf16, const float* act_scale,
                       const int32_t* slot_to_row, void* a_codes, void* a_sf, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !slot_to_row || !a_codes || !a_sf) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && !act_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(a_codes) || !aligned16(a_sf)) return MOE_ERR_INVALID_ARG;
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

moe_status moe_forward_gateup(const moe_config* cfg, int64_t T, const void* packed, const void* a_codes,
                              const void* a_sf, const float* act_scale, const float* inter_scale,
                              const int32_t* expert_offsets, const int32_t* expert_counts, void* h_codes,
                              void* h_sf, float* gateup_debug, uint32_t* status_word, void* stream) {
  moe_status s = gemm_common(cfg, T, packed, expert_offsets, expert_counts);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!a_codes || !a_sf || !h_codes || !h_sf) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && (!act_scale || !inter_scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(h_codes) || !aligned16(h_sf)) return MOE_ERR_INVALID_ARG;
  if (gateup_debug && !aligned16(gateup_debug)) return MOE_ERR_INVALID_ARG;
  moe_weights_layout L;
  layout(cfg, &L);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  moe::GemmLaunch g{};
  g.fmt = cfg->fmt;
  g.gateup = true;
  g.E = cfg->num_experts;
  g.K = cfg->d_model;
  g.n_rows_b = 2 * cfg->d_ffn;
  g.R_max = max_rows(cfg, T);
  g.a_codes = static_cast<const uint8_t*>(a_codes);
  g.a_sf = static_cast<const uint8_t*>(a_sf);
  g.b_codes = base + L.w13_codes;
  g.b_sf = base + L.w13_sf;
  g.offsets = expert_offsets;
  g.counts = expert_counts;
  g.a_scale = act_scale;
  g.w_scales = reinterpret_cast<const float*>(base + L.scales);
  g.h_scale = inter_scale;
  g.h_codes = static_cast<uint8_t*>(h_codes);
  g.h_sf = static_cast<uint8_t*>(h_sf);
  g.dbg = gateup_debug;
  g.out = nullptr;
  g.status = status_word;
  return from_cuda(moe::launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward_down(const moe_config* cfg, int64_t T, const void* packed, const void* h_codes,
                            const void* h_sf, const float* inter_scale, const int32_t* expert_offsets,
                            const int32_t* expert_counts, void* down_out, uint32_t* status_word, void* stream) {
  moe_status s = gemm_common(cfg, T, packed, expert_offsets, expert_counts);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!h_codes || !h_sf || !down_out) return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && !inter_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h_codes) || !aligned16(h_sf) || !aligned16(down_out)) return MOE_ERR_INVALID_ARG;
  moe_weights_layout L;
  layout(cfg, &L);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  moe::GemmLaunch g{};
  g.fmt = cfg->fmt;
  g.gateup = false;
  g.E = cfg->num_experts;
  g.K = cfg->d_ffn;
  g.n_rows_b = cfg->d_model;
  g.R_max = max_rows(cfg, T);
  g.a_codes = static_cast<const uint8_t*>(h_codes);
  g.a_sf = static_cast<const uint8_t*>(h_sf);
  g.b_codes = base + L.w2_codes;
  g.b_sf = base + L.w2_sf;
  g.offsets = expert_offsets;
  g.counts = expert_counts;
  g.a_scale = inter_scale;
  g.w_scales = reinterpret_cast<const float*>(base + L.scales);
  g.h_scale = nullptr;
  g.out = down_out;
  g.status = status_word;
  return from_cuda(moe::launch_gemm(g, static_cast<cudaStream_t>(stream)));
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

moe_status moe_forward_grouped(const moe_config* cfg, int32_t num_groups, const void* packed, const void* a_codes,
                               const void* a_sf, const float* act_scale, const float* inter_scale,
                               const int32_t* group_offsets, const int32_t* group_counts,
                               const int32_t* group_expert, void* h_codes, void* h_sf, void* down_out,
                               float* gateup_debug, uint32_t* status_word, void* stream) {
  moe_status s = check(cfg);
  if (s != MOE_OK) return s;
  if (num_groups < 0 || num_groups > 1024) return MOE_ERR_UNSUPPORTED;
  if (num_groups == 0) return MOE_OK;
  if (!packed || !a_codes || !a_sf || !group_offsets || !group_counts || !group_expert || !h_codes || !h_sf ||
      !down_out)
    return MOE_ERR_INVALID_ARG;
  if (cfg->fmt == MOE_NVFP4 && (!act_scale || !inter_scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(a_codes) || !aligned16(a_sf) || !aligned16(h_codes) || !aligned16(h_sf) ||
      !aligned16(down_out) || (gateup_debug && !aligned16(gateup_debug)))
    return MOE_ERR_INVALID_ARG;
  moe_weights_layout L;
  layout(cfg, &L);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe::GemmLaunch g{};
  g.fmt = cfg->fmt;
  g.E = num_groups;
  g.offsets = group_offsets;
  g.counts = group_counts;
  g.expert_map = group_expert;
  g.n_weights = cfg->num_experts;
  g.w_scales = reinterpret_cast<const float*>(base + L.scales);
  g.status = status_word;
  // gate/up + SwiGLU + requantized h
  g.gateup = true;
  g.K = cfg->d_model;
  g.n_rows_b = 2 * cfg->d_ffn;
  g.a_codes = static_cast<const uint8_t*>(a_codes);
  g.a_sf = static_cast<const uint8_t*>(a_sf);
  g.b_codes = base + L.w13_codes;
  g.b_sf = base + L.w13_sf;
  g.a_scale = act_scale;
  g.h_scale = inter_scale;
  g.h_codes = static_cast<uint8_t*>(h_codes);
  g.h_sf = static_cast<uint8_t*>(h_sf);
  g.dbg = gateup_debug;
  cudaError_t err = moe::launch_gemm(g, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  // down
  g.gateup = false;
  g.K = cfg->d_ffn;
  g.n_rows_b = cfg->d_model;
  g.a_codes = static_cast<const uint8_t*>(h_codes);
  g.a_sf = static_cast<const uint8_t*>(h_sf);
  g.b_codes = base + L.w2_codes;
  g.b_sf = base + L.w2_sf;
  g.a_scale = inter_scale;
  g.h_scale = nullptr;
  g.h_codes = nullptr;
  g.h_sf = nullptr;
  g.dbg = nullptr;
  g.out = down_out;
  return from_cuda(moe::launch_gemm(g, st));
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
