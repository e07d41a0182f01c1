"""Top-k routing, softmax over the selected experts and the token-slot sort.

Test infrastructure only; see the package docstring.

Pages: "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview,
and "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
section "NVFP4 and MXFP8 experts": every decoder layer sends each token to 8
of 384 routed experts, with no shared expert.  The pages do not print the
scoring function; the reading used here (and by the CUDA library) is:
  * router logits are float32 inputs, one row of E per token;
  * the k selected experts are the k largest logits, ties to the lower
    expert index, -0 equal to +0, returned in rank order;
  * the weights are a softmax over the k selected logits, in float32:
      m = l_0, e_j = exp_own(l_j - m), s = ((e_0 + e_1) + e_2) + ...,
      w_j = e_j / s;
  * exp_own is Cody-Waite range reduction plus a degree-7 Taylor polynomial
    in float32, each operation rounded once (no fused multiply-add), so both
    implementations produce the same bits (exp_own below);
  * the slots of each expert are stored in ascending token order, and each
    expert's segment starts at a multiple of 128 rows.
"""

import math

import numpy as np

F32 = np.float32

# Cody-Waite constants.  LN2_HI keeps only 16 significant bits so that
# n * LN2_HI is exact in float32 for |n| < 2^8.
LOG2E_F32 = F32(1.4426950408889634)
LN2_HI_F32 = F32(0.693145751953125)              # 0x3F317200
LN2_LO_F32 = F32(math.log(2.0) - 0.693145751953125)
#: Taylor coefficients 1/i! for i = 0..7, rounded to float32
EXP_TAYLOR_F32 = tuple(F32(1.0 / math.factorial(i)) for i in range(8))
#: below this argument exp_own returns 0 (keeps every result a normal float32)
EXP_UNDERFLOW_F32 = F32(-80.0)

ROW_ALIGN = 128


def exp_own(x):
    """exp(x) for float32 x <= 0 by Cody-Waite reduction and Taylor series.

      n = rint(x * log2(e))                          (ties to even)
      r = (x - n * LN2_HI) - n * LN2_LO
      p = Horner(1/7!, ..., 1/1!, 1/0!) at r         (multiply, then add)
      exp(x) = p * 2^n
    Arguments below -80 return 0.  Every operation is one float32 rounding.

    Follows the reading that the k selected experts are weighted by a softmax of their logits (the pages route
    each token to 8 of 384 experts: "thinkingmachines/Inkling-2-Small", section Overview; "Thinking Machines
    releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts"); the method is Cody
    and Waite's range reduction (Software Manual for the Elementary Functions, 1980) with a Taylor polynomial.
    """
    x = np.asarray(x, dtype=np.float32)
    n = np.rint((x * LOG2E_F32).astype(np.float32)).astype(np.float32)
    r = (x - (n * LN2_HI_F32).astype(np.float32)).astype(np.float32)
    r = (r - (n * LN2_LO_F32).astype(np.float32)).astype(np.float32)
    p = np.full(x.shape, EXP_TAYLOR_F32[7], dtype=np.float32)
    for i in range(6, -1, -1):
        p = ((p * r).astype(np.float32) + EXP_TAYLOR_F32[i]).astype(np.float32)
    two_n = np.exp2(np.clip(n, -126, 127).astype(np.float64)).astype(np.float32)
    out = (p * two_n).astype(np.float32)
    return np.where(x < EXP_UNDERFLOW_F32, F32(0.0), out).astype(np.float32)


def topk_select(logits, k):
    """Indices of the k largest logits per row, ties to the lower index.

    Selection by definition: k rounds, each taking the largest remaining
    value (numpy argmax returns the first, i.e. lowest, index among equal
    maxima, and compares -0 equal to +0).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview (384 routed experts, top-8) and
    "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts"
    (8 of 384 experts per token).
    """
    logits = np.asarray(logits, dtype=np.float32)
    if np.any(np.isnan(logits)):
        raise ValueError("NaN router logit")
    T, E = logits.shape
    work = logits.astype(np.float64).copy()
    ids = np.zeros((T, k), dtype=np.int32)
    for j in range(k):
        best = np.argmax(work, axis=1)
        ids[:, j] = best
        work[np.arange(T), best] = -np.inf
    return ids


def topk_softmax(logits, ids):
    """Softmax over the selected logits (float32, sequential sum in rank order).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts"; the softmax over the k selected
    logits is the reading of the router's weights.
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, k = ids.shape
    sel = np.take_along_axis(logits, ids.astype(np.int64), axis=1).astype(np.float32)
    m = sel[:, :1]
    e = exp_own((sel - m).astype(np.float32))
    s = e[:, 0].astype(np.float32)
    for j in range(1, k):
        s = (s + e[:, j]).astype(np.float32)
    return (e / s[:, None]).astype(np.float32)


def round_up(v, m):
    """Smallest multiple of m that is >= v (v >= 0, m > 0)."""
    return (v + m - 1) // m * m


def sort_slots(ids, num_experts):
    """Counting sort of the T*k token slots by (expert, token).

    Slot t*k + j is token t's j-th choice.  Returns
      counts        int32[E]     slots per expert
      offsets       int32[E+1]   first row of each expert; each segment padded
                                 to a multiple of 128 rows
      sorted_slots  int32[R]     slot stored in each row, -1 for padding,
                                 R = offsets[E]
      slot_to_row   int32[T*k]   inverse map

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and
    MXFP8 experts": each token's 8 expert slots, grouped by expert for the per-expert GEMMs.
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.zeros(num_experts, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    for e in range(num_experts):
        offsets[e + 1] = offsets[e] + round_up(counts[e], ROW_ALIGN)
    R = int(offsets[num_experts])
    sorted_slots = np.full(R, -1, dtype=np.int64)
    slot_to_row = np.zeros(T * k, dtype=np.int64)
    fill = offsets[:-1].copy()
    for s in range(T * k):              # ascending slot order == ascending token order
        e = flat[s]
        row = fill[e]
        fill[e] += 1
        sorted_slots[row] = s
        slot_to_row[s] = row
    return (counts.astype(np.int32), offsets.astype(np.int32),
            sorted_slots.astype(np.int32), slot_to_row.astype(np.int32))


def router_logits(x, w_router):
    """Router scores of every token for every routed expert:
        logits[t, e] = sum_h x[t, h] * W_r[e, h]
    x [T, H] and W_r [E, H] hold bfloat16 values (passed exactly, widened to
    float32 or float64).  Each product is exact in float64 (two 8-bit
    significands); the sum is taken in float64 and rounded once to float32.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview (each token scored against the 384
    routed experts, top-8 kept) and "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
    section "NVFP4 and MXFP8 experts" (8 of 384 experts per token).  The pages do not print the router; the
    reading used is a bias-free linear projection of the layer input, bfloat16 weights, one float32 score per
    expert.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    return (x64 @ w64.T).astype(np.float32)


def router_route(x, w_router, k, num_experts):
    """Routing of tokens from their layer input: the router scores, then route().

    Follows the same passages as router_logits and route.
    """
    return route(router_logits(x, w_router), k, num_experts)


def route(logits, k, num_experts):
    """Whole routing step: top-k ids, softmax weights and the slot sort.

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    ids = topk_select(logits, k)
    w = topk_softmax(logits, ids)
    counts, offsets, sorted_slots, slot_to_row = sort_slots(ids, num_experts)
    return dict(topk_ids=ids, topk_w=w, counts=counts, offsets=offsets,
                sorted_slots=sorted_slots, slot_to_row=slot_to_row)
