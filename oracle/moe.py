"""Permute, expert FFN and combine of the routed MoE layer (oracle side).

Test infrastructure only; see the package docstring.

Pages: "Thinking Machines releases Inkling 2 Small weights under Apache
2.0", section "NVFP4 and MXFP8 experts" (each token goes to 8 of 384
experts; expert activations are quantized to the layer's weight format) and
section TL;DR (the NVFP4 4-vs-6 quantizer).  The expert network is not
printed on the pages; the reading used is a SwiGLU FFN without biases:
    g = x W_gate^T,  u = x W_up^T,  h = silu(g) * u,  o = h W_down^T
with W_gate, W_up of shape [d_ffn, d_model] and W_down of shape
[d_model, d_ffn].  The layer output is y[t] = sum_j w[t, j] * o[row(t, j)].

Arithmetic: quantized operands are dequantized exactly (products of a code,
a block scale and a float32 tensor scale are exact in float64); GEMMs,
SwiGLU and the combine run in float64; h is rounded to float32 before it is
requantized (that requantization is the method's float32 arithmetic), and y
is rounded once to bfloat16.
"""

import numpy as np

from . import formats as fm
from . import route as rt

NVFP4 = "nvfp4"
MXFP8 = "mxfp8"


# --------------------------------------------------------------------------
# quantized tensors: (codes[rows, K], scales[rows, K/block], tensor scale)
# --------------------------------------------------------------------------

def quantize_rows(x, fmt, s_g=None):
    """Quantize float32 rows along K in the layer format.

    NVFP4 uses the 4-vs-6 quantizer with tensor scale s_g; MXFP8 ignores s_g.
    Returns (codes, scales).

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and
    MXFP8 experts": activations are quantized to the layer's weight format; page
    "thinkingmachines/Inkling-2-Small", section Overview: NVFP4 in layers 0-39, MXFP8 in 40-47.
    """
    if fmt == NVFP4:
        return fm.nvfp4_quantize_rows(x, s_g)
    if fmt == MXFP8:
        return fm.mxfp8_quantize_rows(x)
    raise ValueError(fmt)


def dequantize_rows(codes, scales, fmt, s_g=None):
    """Exact float64 values of quantized rows in the layer format (inverse of quantize_rows).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    if fmt == NVFP4:
        return fm.nvfp4_dequantize_rows(codes, scales, s_g)
    if fmt == MXFP8:
        return fm.mxfp8_dequantize_rows(codes, scales)
    raise ValueError(fmt)


def weight_tensor_scale(w, fmt):
    """Per-(expert, matrix) tensor scale: amax / 2688 for NVFP4, 1 for MXFP8.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section TL;DR.
    """
    if fmt == NVFP4:
        return fm.nvfp4_tensor_scale(np.max(np.abs(np.asarray(w, dtype=np.float32))))
    return np.float32(1.0)


def quantize_expert(w_gate, w_up, w_down, fmt):
    """Offline quantization of one expert's three float32 matrices.

    Returns a dict with, for m in ('gate', 'up', 'down'), the codes
    [rows, K], the block-scale codes [rows, K/block] and the tensor scale.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section TL;DR: the experts' weights in NVFP4 (4-vs-6) or MXFP8.
    """
    out = {}
    for name, w in (("gate", w_gate), ("up", w_up), ("down", w_down)):
        s = weight_tensor_scale(w, fmt)
        c, sf = quantize_rows(np.asarray(w, dtype=np.float32), fmt, s)
        out[name] = (c, sf, np.float32(s))
    return out


def dequantize_expert(q, fmt):
    """Exact float64 values of one expert's three quantized matrices.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section TL;DR.
    """
    return {m: dequantize_rows(c, sf, fmt, s) for m, (c, sf, s) in q.items()}


# --------------------------------------------------------------------------
# the steps of the layer
# --------------------------------------------------------------------------

def permute_quantize(x, sorted_slots, k, fmt, s_x=None):
    """Rows of the expert-sorted activation matrix, quantized.

    Row r holds token sorted_slots[r] // k; padding rows (slot -1) are left
    out of the result (returned mask is False there).  Every copy of a token
    is the same quantization of x[t], so it is computed once per token.

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and
    MXFP8 experts": the quantization of the expert inputs is part of the kernel that produces them, so every
    copy of a token is the same quantization.
    """
    x = np.asarray(x, dtype=np.float32)
    codes_t, sf_t = quantize_rows(x, fmt, s_x)
    valid = sorted_slots >= 0
    tok = np.where(valid, sorted_slots // k, 0)
    return codes_t[tok], sf_t[tok], valid


def swiglu(g, u):
    """silu(g) * u = g * u / (1 + exp(-g)) in float64.

    For g below about -709 exp(-g) overflows to inf and the quotient is the
    limit, a signed zero; numpy's overflow warning is silenced for that case.

    Follows the expert FFN; the pages do not print it, SwiGLU without bias is the reading.
    """
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g * u / (1.0 + np.exp(-g))


def expert_ffn(a_deq, wq_deq, fmt, s_h):
    """One expert on its rows: GEMM1 -> SwiGLU -> requantize h -> GEMM2.

    a_deq  float64 [m, H]   dequantized activation rows
    wq_deq dict of float64 dequantized weights
    Returns dict(gate=[m, I], up=[m, I] float64, h_codes, h_sf, out=[m, H]).

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and
    MXFP8 experts": the intermediate is requantized to the layer's format before the down projection.
    """
    g = a_deq @ wq_deq["gate"].T
    u = a_deq @ wq_deq["up"].T
    h = swiglu(g, u).astype(np.float32)
    h_codes, h_sf = quantize_rows(h, fmt, s_h)
    h_deq = dequantize_rows(h_codes, h_sf, fmt, s_h)
    out = h_deq @ wq_deq["down"].T
    return dict(gate=g, up=u, h=h, h_codes=h_codes, h_sf=h_sf, out=out)


def combine(out_rows, topk_w, slot_to_row):
    """y[t] = sum_j w[t, j] * out[slot_to_row[t*k + j]] in float64, then bf16.

    Follows page "thinkingmachines/Inkling-2-Small", section Overview: routed experts only, no shared expert.
    """
    T, k = topk_w.shape
    y = np.zeros((T, out_rows.shape[1]), dtype=np.float64)
    for j in range(k):
        rows = slot_to_row.reshape(T, k)[:, j]
        y += topk_w[:, j].astype(np.float64)[:, None] * out_rows[rows]
    return fm.bf16_round(y)


def forward(x, logits, experts_q, k, fmt, s_x=None, s_h=None, num_experts=None):
    """Whole layer: route -> permute+quantize -> per-expert FFN -> combine.

    x          float32 [T, H] (the bf16 input, widened exactly)
    logits     float32 [T, E]
    experts_q  dict e -> quantize_expert(...) result, for every expert that
               receives a slot (others may be missing)
    Returns a dict with every intermediate: the routing tensors, A codes /
    scales per row, gate/up float64 per row, h codes / scales per row, the
    per-row down output and y.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview, "Thinking Machines releases Inkling 2
    Small weights under Apache 2.0", section TL;DR and "Thinking Machines releases Inkling 2 Small weights
    under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    E = num_experts if num_experts is not None else logits.shape[1]
    r = rt.route(logits, k, E)
    a_codes, a_sf, valid = permute_quantize(x, r["sorted_slots"], k, fmt, s_x)
    R = r["sorted_slots"].shape[0]
    res = dict(r)
    res.update(a_codes=a_codes, a_sf=a_sf, valid=valid)
    I = None
    out_rows = np.zeros((R, H), dtype=np.float64)
    gate = up = h_codes = h_sf = None
    for e in range(E):
        lo, cnt = int(r["offsets"][e]), int(r["counts"][e])
        if cnt == 0:
            continue
        wq = dequantize_expert(experts_q[e], fmt)
        a_deq = dequantize_rows(a_codes[lo:lo + cnt], a_sf[lo:lo + cnt], fmt, s_x)
        f = expert_ffn(a_deq, wq, fmt, s_h)
        if I is None:
            I = f["gate"].shape[1]
            gate = np.zeros((R, I)); up = np.zeros((R, I))
            h_codes = np.zeros((R, I), dtype=np.uint8)
            h_sf = np.zeros((R, f["h_sf"].shape[1]), dtype=np.uint8)
        gate[lo:lo + cnt] = f["gate"]
        up[lo:lo + cnt] = f["up"]
        h_codes[lo:lo + cnt] = f["h_codes"]
        h_sf[lo:lo + cnt] = f["h_sf"]
        out_rows[lo:lo + cnt] = f["out"]
    y = combine(out_rows, r["topk_w"], r["slot_to_row"])
    res.update(gate=gate, up=up, h_codes=h_codes, h_sf=h_sf, out=out_rows, y=y)
    return res


def forward_tokens(x_rows, logits_rows, experts_q, k, fmt, s_x=None, s_h=None):
    """Layer output for a few tokens, one at a time (for sampled checks).

    The same steps as forward(), applied to each given token on its own:
    top-k, softmax, quantize x[t], the k expert FFNs, weighted sum, bf16.
    experts_q must hold every expert these tokens select.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview, "Thinking Machines releases Inkling 2
    Small weights under Apache 2.0", section TL;DR and "Thinking Machines releases Inkling 2 Small weights
    under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    x_rows = np.asarray(x_rows, dtype=np.float32)
    logits_rows = np.asarray(logits_rows, dtype=np.float32)
    ids = rt.topk_select(logits_rows, k)
    w = rt.topk_softmax(logits_rows, ids)
    codes, sf = quantize_rows(x_rows, fmt, s_x)
    a_deq = dequantize_rows(codes, sf, fmt, s_x)
    y = np.zeros(x_rows.shape, dtype=np.float64)
    cache = {}
    for t in range(x_rows.shape[0]):
        for j in range(k):
            e = int(ids[t, j])
            if e not in cache:
                cache[e] = dequantize_expert(experts_q[e], fmt)
            f = expert_ffn(a_deq[t:t + 1], cache[e], fmt, s_h)
            y[t] += float(w[t, j]) * f["out"][0]
    return dict(topk_ids=ids, topk_w=w, a_codes=codes, a_sf=sf, y=fm.bf16_round(y))


# --------------------------------------------------------------------------
# BF16 experts with LoRA adapters
# --------------------------------------------------------------------------

def lora_project(a, w, lora_a, lora_b, scaling):
    """a W^T + scaling * (a A^T) B^T in float64: a projection with weight
    W [N, K] and a rank-r adapter A [r, K], B [N, r].

    Follows page "thinkingmachines/Inkling-2-Small", section Configurations, and page "Thinking Machines
    releases Inkling 2 Small weights under Apache 2.0", section "LoRA and reinforcement learning": adapters on
    the routed experts need BF16 expert weights (a rank-32 adapter in the pages' validation run).  The adapter
    form is the usual low-rank update W + scaling * B A, applied without merging.
    """
    a = np.asarray(a, dtype=np.float64)
    out = a @ np.asarray(w, dtype=np.float64).T
    if lora_a is None:
        return out
    z = a @ np.asarray(lora_a, dtype=np.float64).T
    return out + float(scaling) * (z @ np.asarray(lora_b, dtype=np.float64).T)


def expert_ffn_bf16(a, w, lora, scaling):
    """One BF16 expert with adapters on gate, up and down:
        g = proj(a, gate), u = proj(a, up), h = bf16(silu(g) * u),
        out = proj(h, down)
    a float64 [m, H] (bf16 values); w dict of bf16-valued [I, H] / [H, I]
    matrices; lora dict m -> (A, B) or None.  The intermediate h is the bf16
    input of the down projection, as in a BF16 model.

    Follows the same passages as lora_project; SwiGLU as in expert_ffn.
    """
    lo = lora or {}
    g = lora_project(a, w["gate"], *lo.get("gate", (None, None)), scaling)
    u = lora_project(a, w["up"], *lo.get("up", (None, None)), scaling)
    h = fm.bf16_round(swiglu(g, u))
    out = lora_project(h, w["down"], *lo.get("down", (None, None)), scaling)
    return dict(gate=g, up=u, h=h, out=out)


def forward_bf16(x, logits, experts_w, experts_lora, k, scaling, num_experts=None):
    """Whole layer with BF16 experts and adapters: route -> per-expert FFN on
    the rows of its tokens (no quantization) -> combine.

    experts_w[e] dict of gate/up/down bf16-valued matrices; experts_lora[e]
    dict m -> (A, B), or None for an expert without adapters.

    Follows the same passages as lora_project, and route / combine.
    """
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    E = num_experts if num_experts is not None else logits.shape[1]
    r = rt.route(logits, k, E)
    R = r["sorted_slots"].shape[0]
    out_rows = np.zeros((R, H), dtype=np.float64)
    gate = up = hb = None
    for e in range(E):
        lo, cnt = int(r["offsets"][e]), int(r["counts"][e])
        if cnt == 0:
            continue
        tok = r["sorted_slots"][lo:lo + cnt] // k
        f = expert_ffn_bf16(x[tok].astype(np.float64), experts_w[e], experts_lora.get(e), scaling)
        if gate is None:
            I = f["gate"].shape[1]
            gate, up, hb = np.zeros((R, I)), np.zeros((R, I)), np.zeros((R, I))
        gate[lo:lo + cnt], up[lo:lo + cnt], hb[lo:lo + cnt] = f["gate"], f["up"], f["h"]
        out_rows[lo:lo + cnt] = f["out"]
    y = combine(out_rows, r["topk_w"], r["slot_to_row"])
    res = dict(r)
    res.update(gate=gate, up=up, h=hb, out=out_rows, y=y)
    return res
