/*
 * moe_b200.h -- C ABI of the routed Mixture-of-Experts expert layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer is the expert half of an Inkling 2 Small decoder layer: every
 * token is sent to top_k of num_experts routed experts (384 and 8 in the
 * model; no shared expert), each expert is a SwiGLU FFN whose weights are
 * NVFP4 (layers 0-39) or MXFP8 (layers 40-47), and the activations entering
 * each GEMM are quantized to the weight format inside the kernel that
 * produces them.  Sources, by page and section:
 *   [P1] "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview:
 *        384 routed experts, top-8, no shared experts; NVFP4 experts in
 *        layers 0-39 and MXFP8 in layers 40-47.
 *   [P2] "Thinking Machines releases Inkling 2 Small weights under Apache
 *        2.0", section TL;DR: the NVFP4 quantizer maps each block's maximum
 *        to both 4 and 6 and keeps the lower-error result; section "NVFP4 and
 *        MXFP8 experts": expert activations are quantized to match each
 *        layer's weight format, folded into the kernels that produce them.
 *
 *   [P3] "thinkingmachines/Inkling-2-Small", section Configurations, and
 *        "Thinking Machines releases Inkling 2 Small weights under Apache
 *        2.0", section "LoRA and reinforcement learning": adapters on the
 *        routed experts need BF16 expert weights (a rank-32 adapter in the
 *        pages' validation run).
 *
 * One layer on one stream is
 *     moe_route_topk -> moe_permute -> moe_forward -> moe_unpermute_combine
 * with moe_quantize_weights run once, offline.
 *
 * Conventions shared by every call
 *   - Memory: every pointer argument is DEVICE memory allocated by the caller
 *     (for example a PyTorch tensor's data_ptr()), unless stated otherwise.
 *     The library never allocates, frees or keeps device memory and keeps no
 *     pointer after a call returns.  Pointers must be 16-byte aligned.
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream)
 *     of the current device, where the work is launched; a stream of
 *     another device is not supported (moe_route_topk_noalloc refuses it
 *     with MOE_ERR_INVALID_ARG, the Python binding refuses it for every
 *     call).
 *     Every call only enqueues work: nothing blocks the host and nothing is
 *     copied back to the host, so the whole layer can be captured in a CUDA
 *     graph.  Device-side scalars (activation scales) are read on the device.
 *   - Errors: arguments are validated on the host before anything is
 *     enqueued and reported as a moe_status; a failed launch returns
 *     MOE_ERR_CUDA.  Kernels never trap: every wait is bounded, and a wait
 *     that runs out sets a bit of the optional device status word (see
 *     MOE_DEVICE_*), which the caller reads after synchronizing.
 *   - Supported shapes: d_model % 256 == 0, d_ffn % 128 == 0, 1 <= top_k <=
 *     min(8, num_experts), 1 <= num_experts <= 1024, 0 <= T <= 2^20.
 *   - Layout of quantized operands.  A code row holds K codes: NVFP4 packs
 *     two E2M1 codes per byte, element 2i in the low nibble of byte i; MXFP8
 *     stores one E4M3 code per byte.  Zero codes are always the +0 code.  Each
 *     row is padded to kb = roundup(K * bits / 8, 128) bytes.  A [rows, kb]
 *     code matrix is stored tiled, ready to copy into the tensor core's
 *     shared-memory operand layout: tiles of TR rows x 128 bytes, K tile
 *     fastest (tile (row / TR, byte / 128) at ((row / TR) * (kb / 128) +
 *     byte / 128) * TR * 128), and inside a tile row r = row % TR at r * 128
 *     with its 16-byte chunk c = (byte % 128) / 16 at chunk position
 *     c ^ (r % 8) (the 128-byte swizzle).  TR = 256 for weights and 128 for
 *     activations (permuted x and the intermediate h).  Block scales are
 *     stored in 512-byte atoms of 128 rows x 4 scale columns (see
 *     moe_sf_offset()).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad size */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside the supported set */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than the size query says */
  MOE_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} moe_status;

typedef enum {
  MOE_NVFP4 = 0, /* E2M1 codes, 16-element E4M3 block scales, fp32 tensor scale [P1, P2] */
  MOE_MXFP8 = 1, /* E4M3 codes, 32-element E8M0 block scales [P1] */
  MOE_BF16 = 2   /* bf16 expert weights and activations, with LoRA adapters on the
                    experts (rank <= 32) [P3] */
} moe_format;

typedef struct {
  int32_t num_experts; /* E: routed experts (384) */
  int32_t top_k;       /* k: experts per token (8) */
  int32_t d_model;     /* H: hidden size (4096) */
  int32_t d_ffn;       /* I: expert intermediate size (2560) */
  int32_t fmt;         /* moe_format of the weights and activations */
} moe_config;

/* Bits of the optional device status word (uint32, caller-owned, zeroed by
 * the caller).  A set bit means a kernel gave up on a wait and its outputs
 * are incomplete. */
#define MOE_DEVICE_TIMEOUT_PRODUCER 0x1u
#define MOE_DEVICE_TIMEOUT_MMA 0x2u
#define MOE_DEVICE_TIMEOUT_EPILOGUE 0x4u
#define MOE_DEVICE_TIMEOUT_SELFTEST 0x8u
/* moe_forward_grouped: a group named an expert outside the packed weights
 * (expert 0's weights were used for its rows instead). */
#define MOE_DEVICE_BAD_GROUP_EXPERT 0x10u

/* Layout of the packed expert weights (byte offsets from the buffer start).
 * For NVFP4 (bits = 4, sfvec = 16) and MXFP8 (bits = 8, sfvec = 32), with
 * kb(K) = roundup(K * bits / 8, 128) and code matrices tiled with TR = 256:
 *   w13_codes  [E][2I x kb(H)]    gate and up rows interleaved in groups of
 *                                 32: row 64g + i is gate channel 32g + i and
 *                                 row 64g + 32 + i is up channel 32g + i
 *   w13_sf     [E][2I*H/sfvec]    block scales of w13, atom layout per expert
 *   w2_codes   [E][H x kb(I)]     down projection, one row per output channel
 *   w2_sf      [E][H*I/sfvec]     block scales of w2, atom layout per expert
 *   scales     [E][3] float32     tensor scales of (gate, up, down); 1.0 for
 *                                 MXFP8
 */
/* MOE_BF16 (no quantization; one extra 64-element K tile per row carries
 * the adapters, so kb(K) = 2K + 128):
 *   w13_codes  [E][2I x kb(H)]    bf16 rows as above (gate / up interleaved);
 *                                 the last K tile of a gate row holds
 *                                 B_gate[c][0..32) then 32 zeros, of an up row
 *                                 32 zeros then B_up[c][0..32)
 *   w13_sf     [E][64 x 2H]       the adapters' A_gate (rows 0-31) and A_up
 *                                 (rows 32-63), bf16, tiled with TR = 64
 *   w2_codes   [E][H x kb(I)]     bf16 down rows; last K tile B_down[n][0..32)
 *                                 then 32 zeros
 *   w2_sf      [E][64 x 2I]       A_down (rows 0-31) and 32 zero rows, TR = 64
 *   scales     [E][3] float32     (adapter scaling, 0, 0)
 * An adapter of rank r < 32 is zero-padded; an expert without one has zeros. */
typedef struct {
  int64_t w13_codes;
  int64_t w13_sf;
  int64_t w2_codes;
  int64_t w2_sf;
  int64_t scales;
  int64_t total_bytes;
} moe_weights_layout;

/* ---------------------------------------------------------------- sizes */

/* Validate a configuration.  Returns MOE_OK if the library supports it. */
MOE_API moe_status moe_check_config(const moe_config* cfg);

/* Byte offsets of the parts of the packed weight buffer (see above). */
MOE_API moe_status moe_get_weights_layout(const moe_config* cfg, moe_weights_layout* out);

/* Upper bound R_max on the number of permuted rows for T tokens: every
 * expert's segment is padded to a multiple of 128 rows, so
 * R_max = roundup128(T*k + 127*min(E, T*k)).  Returns -1 on a bad config. */
MOE_API int64_t moe_max_rows(const moe_config* cfg, int64_t T);

/* Bytes of the (tiled) quantized codes / block scales of `rows` rows of
 * length K in the configured format (K = d_model for the permuted activations
 * A, K = d_ffn for the intermediate h; rows a multiple of 128).  Returns -1
 * on a bad argument. */
MOE_API int64_t moe_codes_bytes(const moe_config* cfg, int64_t rows, int64_t K);
MOE_API int64_t moe_sf_bytes(const moe_config* cfg, int64_t rows, int64_t K);

/* Byte offset of the block scale of (row, scale column) in a scale buffer of
 * rows x nsf scale columns (nsf = K/16 for NVFP4, K/32 for MXFP8, a multiple
 * of 4): atoms of 128 rows x 4 columns, K direction fastest; inside an atom
 * byte (row % 32) * 16 + ((row % 128) / 32) * 4 + col % 4. */
MOE_API int64_t moe_sf_offset(int64_t row, int64_t col, int64_t nsf);

/* Workspace bytes moe_route_topk needs for T tokens. */
MOE_API int64_t moe_route_workspace_bytes(const moe_config* cfg, int64_t T);

/* ---------------------------------------------------------------- calls */

/* Offline expert-weight quantization [P1 Overview; P2 TL;DR and "NVFP4 and
 * MXFP8 experts"].  Quantizes experts [expert_begin, expert_begin +
 * expert_count) into the packed buffer `packed` (moe_get_weights_layout;
 * other experts are left untouched, so the whole model can be quantized a
 * slice at a time).
 *   w_gate, w_up  float32 [expert_count][I][H] (row-major, K = H contiguous)
 *   w_down        float32 [expert_count][H][I]
 * NVFP4: the tensor scale of each (expert, matrix) is amax / 2688 (1 when the
 * matrix is all zero) and every 16-element block along K takes the 4-vs-6
 * scale pick.  MXFP8: 32-element blocks with the OCP shared exponent, tensor
 * scales 1.  Inputs must be finite. */
MOE_API moe_status moe_quantize_weights(const moe_config* cfg, int32_t expert_begin, int32_t expert_count,
                                const float* w_gate, const float* w_up, const float* w_down, void* packed,
                                void* stream);

/* Offline packing of BF16 expert weights and their LoRA adapters [P3]
 * (MOE_BF16 only; moe_quantize_weights returns MOE_ERR_UNSUPPORTED for it).
 * Experts [expert_begin, expert_begin + expert_count) of `packed`:
 *   w_gate, w_up    bf16 [n][I][H];  w_down  bf16 [n][H][I]
 *   lora_a_gate, lora_a_up  bf16 [n][lora_rank][H]; lora_a_down bf16
 *                   [n][lora_rank][I]; lora_b_gate, lora_b_up bf16
 *                   [n][I][lora_rank]; lora_b_down bf16 [n][H][lora_rank]
 *                   (all six, or all six NULL for experts without adapters)
 *   lora_rank       1 .. 32 (MOE_ERR_UNSUPPORTED otherwise)
 *   lora_scaling    the adapters' scaling (alpha / rank)
 * Each projection then computes W a + lora_scaling * B (A a).  The adapters'
 * products A a are rounded to bf16 (they feed the tensor cores as bf16 with
 * the expert's own rows). */
MOE_API moe_status moe_pack_weights_bf16(const moe_config* cfg, int32_t expert_begin, int32_t expert_count,
                                         const void* w_gate, const void* w_up, const void* w_down,
                                         const void* lora_a_gate, const void* lora_b_gate, const void* lora_a_up,
                                         const void* lora_b_up, const void* lora_a_down, const void* lora_b_down,
                                         int32_t lora_rank, float lora_scaling, void* packed, void* stream);

/* Routing [P1 Overview; P2 "NVFP4 and MXFP8 experts": top-k of the routed
 * experts, no shared expert].  For T tokens of float32 logits [T][E]:
 *   topk_ids       int32 [T][k]   the k largest logits, ties to the lower
 *                                 expert index, in rank order
 *   topk_w         float32 [T][k] softmax over the k selected logits:
 *                                 m = l_0, e_j = exp(l_j - m), w_j = e_j /
 *                                 (((e_0 + e_1) + e_2) + ...), float32, with
 *                                 exp by Cody-Waite reduction and a degree-7
 *                                 Taylor polynomial (one rounding per step;
 *                                 arguments below -80 give 0)
 *   expert_counts  int32 [E]      slots routed to each expert
 *   expert_offsets int32 [E+1]    first row of each expert; every segment is
 *                                 padded to a multiple of 128 rows;
 *                                 expert_offsets[E] = rows in use
 *   sorted_slots   int32 [R_max]  slot t*k+j held by each row, rows of one
 *                                 expert in ascending token order; -1 for
 *                                 padding rows and rows >= expert_offsets[E]
 *                                 (R_max = 0 when T = 0: may then be NULL)
 *   slot_to_row    int32 [T*k]    row of each slot
 *   workspace      moe_route_workspace_bytes(cfg, T) bytes of scratch
 * Logits must not be NaN.  The result does not depend on thread timing. */
MOE_API moe_status moe_route_topk(const moe_config* cfg, int64_t T, const float* logits, int32_t* topk_ids,
                          float* topk_w, int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_slots,
                          int32_t* slot_to_row, void* workspace, int64_t workspace_bytes, void* stream);

/* Routing from the layer input, with the router scores fused into the
 * top-k [P1 Overview; P2 "NVFP4 and MXFP8 experts": each token is scored
 * against the routed experts and sent to the top_k best].  The scores
 *     logits[t][e] = sum_h x[t][h] * w_router[e][h]
 * are computed on the tensor cores (bf16 products, float32 accumulation) and
 * reduced to the k selected experts in the same kernel; they reach memory only
 * through the optional logits_out.  Then, exactly as moe_route_topk does for
 * given logits: top-k (ties to the lower index, rank order), the softmax over
 * the k selected scores, counts, padded offsets and the slot sort.
 *   x_bf16         bf16 [T][d_model], row-major (the layer input)
 *   w_router_bf16  bf16 [num_experts][d_model], row-major (no bias)
 *   logits_out     optional float32 [T][num_experts]: a copy of the scores
 *                  (NULL in normal use)
 *   other outputs and workspace as for moe_route_topk (same sizes)
 *   status_word    optional uint32 device status word (MOE_DEVICE_*)
 * Supported: num_experts <= 512 (MOE_ERR_UNSUPPORTED otherwise).  The
 * float32 sums are taken in the tensor core's order, so a score can differ
 * from the exactly rounded sum in its last bits; results do not depend on
 * thread timing.  Batches of up to 37 tiles of 128 tokens (with at most 384
 * experts) split d_model over a cluster of 4 or 8 CTAs per tile and add the
 * partial sums, on chip, in cluster-rank order.  Batches of up to 74 tiles
 * whose num_experts is a multiple of 128 split the experts over a cluster of
 * two CTAs per tile (each score is still one CTA's full sum). */
MOE_API moe_status moe_router_topk(const moe_config* cfg, int64_t T, const void* x_bf16, const void* w_router_bf16,
                                   float* logits_out, int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                                   int32_t* expert_offsets, int32_t* sorted_slots, int32_t* slot_to_row,
                                   void* workspace, int64_t workspace_bytes, uint32_t* status_word, void* stream);

/* Permute-gather with fused activation quantization [P2 "NVFP4 and MXFP8
 * experts": activations quantized to the weight format inside the producing
 * kernel; P2 TL;DR: the 4-vs-6 pick].  Token t's row x[t] (bf16 [T][H]) is
 * quantized once and written to each of its k rows slot_to_row[t*k+j] of
 *   a_codes  tiled codes, TR = 128 (moe_codes_bytes(cfg, R_max, H))
 *   a_sf     block scales       (moe_sf_bytes(cfg, R_max, H))
 * act_scale: device float32 scalar, the static NVFP4 tensor scale of x
 * (ignored, may be NULL, for MXFP8).  Padding rows are not written. */
MOE_API moe_status moe_permute(const moe_config* cfg, int64_t T, const void* x_bf16, const float* act_scale,
                       const int32_t* slot_to_row, void* a_codes, void* a_sf, void* stream);

/* Expert FFN over the permuted rows [P2 "NVFP4 and MXFP8 experts"; SwiGLU]:
 * for the rows of expert e,
 *     g = A W_gate[e]^T * s_a * s_gate[e],  u = A W_up[e]^T * s_a * s_up[e],
 *     h = silu(g) * u  (float32)  -> quantized in the GEMM epilogue to the
 *         layer format (NVFP4 with tensor scale *inter_scale, 4-vs-6)
 *     out = h W_down[e]^T * s_h * s_down[e]  -> bf16 [R_max][H]
 * on tcgen05 block-scaled tensor cores.  `T` bounds the rows in use (they
 * are read from expert_offsets[E] on the device).
 *   packed            weights from moe_quantize_weights
 *   a_codes, a_sf     from moe_permute
 *   act_scale, inter_scale  device float32 scalars (NVFP4; NULL for MXFP8)
 *   expert_offsets, expert_counts  from moe_route_topk
 *   h_codes, h_sf     caller buffers of moe_codes_bytes / moe_sf_bytes(cfg,
 *                     R_max, I): the quantized intermediate
 *   down_out          bf16 [R_max][H]; only rows holding a slot are written
 *   gateup_debug      optional float32 [R_max][2I]: g in columns [0, I) and
 *                     u in [I, 2I) (NULL in normal use)
 *   status_word       optional uint32 device status word (MOE_DEVICE_*)
 * moe_forward runs moe_forward_gateup then moe_forward_down.
 * MOE_BF16 [P3]: no quantization and no block scales (a_sf, h_sf may be
 * NULL, the activation scales are ignored); h is bf16 (moe_codes_bytes(cfg,
 * R_max, I)); moe_forward_gateup first writes each row's adapter product
 * lora_scaling * (A_gate a, A_up a) into the last K tile of a_codes (left
 * free by moe_permute), then the gate/up GEMM, then the down adapter's
 * product of h into h's last K tile; moe_forward_down runs over it. */
MOE_API moe_status moe_forward(const moe_config* cfg, int64_t T, const void* packed, const void* a_codes,
                       const void* a_sf, const float* act_scale, const float* inter_scale,
                       const int32_t* expert_offsets, const int32_t* expert_counts, void* h_codes, void* h_sf,
                       void* down_out, float* gateup_debug, uint32_t* status_word, void* stream);
MOE_API moe_status moe_forward_gateup(const moe_config* cfg, int64_t T, const void* packed, const void* a_codes,
                              const void* a_sf, const float* act_scale, const float* inter_scale,
                              const int32_t* expert_offsets, const int32_t* expert_counts, void* h_codes,
                              void* h_sf, float* gateup_debug, uint32_t* status_word, void* stream);
MOE_API moe_status moe_forward_down(const moe_config* cfg, int64_t T, const void* packed, const void* h_codes,
                            const void* h_sf, const float* inter_scale, const int32_t* expert_offsets,
                            const int32_t* expert_counts, void* down_out, uint32_t* status_word, void* stream);

/* Expert FFN over rows grouped by the expert whose weights they use, for
 * expert parallelism [P1 Overview: expert parallelism follows the TP group]:
 * a rank that holds a slice of the experts receives, from every rank, the
 * rows routed to its experts, each source's rows already grouped by expert
 * and padded to 128 rows.  Row group g (rows group_offsets[g] ..
 * group_offsets[g] + group_counts[g] - 1) is computed exactly as moe_forward
 * computes the rows of expert group_expert[g] of `packed`.
 *   cfg            num_experts = experts held in `packed` (this rank's slice)
 *   num_groups     row groups, 0 .. 1024
 *   max_rows       rows the buffers hold (a multiple of 128, >= the last
 *                  group offset)
 *   group_offsets  int32 [num_groups + 1], device: first row of each group,
 *                  multiples of 128, non-decreasing, group_offsets[0] = 0
 *   group_counts   int32 [num_groups], device: rows in use per group,
 *                  <= group_offsets[g + 1] - group_offsets[g]
 *   group_expert   int32 [num_groups], device: expert of `packed` per group;
 *                  an index outside 0 .. num_experts - 1 is replaced by 0 and
 *                  sets MOE_DEVICE_BAD_GROUP_EXPERT in the status word
 *   a_codes, a_sf, h_codes, h_sf, down_out, gateup_debug, scales, status
 *                  as for moe_forward, sized for group_offsets[num_groups]
 *                  rows (buffers sized by moe_codes_bytes / moe_sf_bytes for a
 *                  multiple of 128 rows at least that large)
 * The row layout and the results of each row are independent of the other
 * groups: a row gives the same bits as in moe_forward. */
MOE_API moe_status moe_forward_grouped(const moe_config* cfg, int32_t num_groups, int64_t max_rows,
                                       const void* packed, const void* a_codes, const void* a_sf, const float* act_scale,
                                       const float* inter_scale, const int32_t* group_offsets,
                                       const int32_t* group_counts, const int32_t* group_expert, void* h_codes,
                                       void* h_sf, void* down_out, float* gateup_debug, uint32_t* status_word,
                                       void* stream);

/* Weighted un-permute and combine [routed experts, no shared expert, P1
 * Overview]: y[t] = sum_{j<k} topk_w[t][j] * down_out[slot_to_row[t*k+j]],
 * accumulated in float32 in rank order, rounded once to bf16 [T][H]. */
MOE_API moe_status moe_unpermute_combine(const moe_config* cfg, int64_t T, const void* down_out, const float* topk_w,
                                 const int32_t* slot_to_row, void* y_bf16, void* stream);

/* Routing for callers that cannot allocate device memory (no counterpart on
 * the source pages; an addition of this library).  Same arguments, results
 * and guarantees as moe_route_topk, bit for bit, without the workspace: its
 * scratch is a fixed 4 MiB array compiled into the library, which every GPU
 * that loads the library keeps until the process exits.  Use it where the
 * caller has only its input and output buffers, for example a plugin inside
 * another runtime or a host that plans all device memory once.
 *   - Limit: moe_route_workspace_bytes(cfg, T) must be <= 4 MiB (for E = 384
 *     that is up to 43,680 tokens); larger sizes return MOE_ERR_WORKSPACE
 *     and enqueue nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) for that device; make that first call outside
 *     any CUDA stream capture.  With CUDA's lazy module loading (the
 *     default) the array's 4 MiB are only then allocated on that device, so
 *     the first call can fail with MOE_ERR_CUDA when the device is out of
 *     memory; later calls reuse the address.
 *   - The work runs on the current device: `stream` must be NULL (the
 *     default stream) or a stream of the current device, else the call
 *     returns MOE_ERR_INVALID_ARG and enqueues nothing.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (different streams, or different host threads) race and may return
 *     wrong results.  Calls on one stream are safe.
 *   - Calls no allocating routine (no cudaMalloc / cudaFree). */
MOE_API moe_status moe_route_topk_noalloc(const moe_config* cfg, int64_t T, const float* logits, int32_t* topk_ids,
                                          float* topk_w, int32_t* expert_counts, int32_t* expert_offsets,
                                          int32_t* sorted_slots, int32_t* slot_to_row, void* stream);

/* Failure-detection self-test (diagnostic; no counterpart on the pages):
 * enqueues one CTA that waits, with the same bounded mbarrier wait the GEMM
 * roles use, on a barrier that nothing ever arrives at.  The wait gives up
 * after limit_ns nanoseconds (1 us .. 5 s) and sets
 * MOE_DEVICE_TIMEOUT_SELFTEST in *status_word (device uint32).  The kernel
 * then returns normally: no trap, no fault, the context stays usable. */
MOE_API moe_status moe_selftest_bounded_wait(uint32_t* status_word, int64_t limit_ns, void* stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
