"""Number formats and block quantizers of the expert layer (oracle side).

Test infrastructure only; see the package docstring.

Formats (the pages name them, the definitions are the OCP MX v1.0 and the
NVFP4 conventions):
  * E2M1: 1 sign bit, 2 exponent bits, 1 mantissa bit; magnitudes
    {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  Encoding is round-to-nearest-even with
    saturation to +-6.
  * E4M3 ("FN" variant): bias 7, no infinities, 0x7F / 0xFF are NaN, largest
    finite value 448, subnormal step 2^-9.  Encoding is round-to-nearest-even
    with saturation to +-448 ("satfinite").
  * E8M0: unsigned power of two 2^(e-127), e in 0..254; 255 is NaN.

Block quantizers
  * NVFP4 (page "Thinking Machines releases Inkling 2 Small weights under
    Apache 2.0", section TL;DR: the block maximum is mapped to both 4 and 6
    and the lower-error result is kept).  16-element blocks along K, one E4M3
    block scale per block, one float32 tensor scale s_g per tensor.  The
    arithmetic is float32 with one rounding per operation (no fused
    multiply-add); the error of a candidate is the sum of squared errors in
    the dequantized domain, summed by the fixed pairwise tree
    ((d0+d1)+(d2+d3))+((d4+d5)+(d6+d7)) ...; candidate 4 wins only when its
    error is strictly lower, so ties go to 6.
  * MXFP8 (page "thinkingmachines/Inkling-2-Small", section Overview: MXFP8
    experts in layers 40-47).  32-element blocks, E4M3 elements, one E8M0
    scale per block chosen by the OCP rule e = floor(log2(amax)) - 8 + 127
    (8 = largest exponent of E4M3), clamped to 0..254; no tensor scale and
    no 4-vs-6 search (the pages describe that search for NVFP4 only).
"""

import numpy as np

F32 = np.float32

# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------

#: magnitude of each 3-bit E2M1 magnitude code
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def e2m1_decode(codes):
    """4-bit E2M1 codes (bit 3 = sign) -> float64 values.

    Follows the E2M1 element type of the NVFP4 experts (pages "thinkingmachines/Inkling-2-Small", section
    Overview; "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8
    experts"); values as the OCP MX v1.0 format definition.
    """
    codes = np.asarray(codes).astype(np.int64)
    mag = np.asarray(E2M1_MAGNITUDES, dtype=np.float64)[codes & 7]
    return np.where((codes >> 3) & 1, -mag, mag)


def e2m1_encode_magnitude(v):
    """Round |v| >= 0 to the nearest E2M1 magnitude, ties to the even code.

    The decision points are the midpoints between neighbouring magnitudes:
    0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.  At a midpoint the code with a zero
    mantissa bit wins (0, 1, 1, 2, 2, 4, 4); anything above 5 saturates to 6.
    Returns the 3-bit magnitude code (0..7).

    Follows the E2M1 element type of the NVFP4 experts (pages "thinkingmachines/Inkling-2-Small", section
    Overview; "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8
    experts"); rounding as the OCP MX v1.0 conversion rule.
    """
    v = np.asarray(v, dtype=np.float64)
    code = np.zeros(v.shape, dtype=np.int64)
    code = np.where(v > 0.25, 1, code)    # (0.25, 0.75)  -> 0.5
    code = np.where(v >= 0.75, 2, code)   # [0.75, 1.25]  -> 1.0
    code = np.where(v > 1.25, 3, code)    # (1.25, 1.75)  -> 1.5
    code = np.where(v >= 1.75, 4, code)   # [1.75, 2.5]   -> 2.0
    code = np.where(v > 2.5, 5, code)     # (2.5, 3.5)    -> 3.0
    code = np.where(v >= 3.5, 6, code)    # [3.5, 5]      -> 4.0
    code = np.where(v > 5.0, 7, code)     # (5, inf)      -> 6.0
    return code


# --------------------------------------------------------------------------
# E4M3 (FN)
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """8-bit E4M3FN codes -> float64 values (NaN for 0x7F and 0xFF).

    Follows E4M3, the element type of the MXFP8 experts and the block-scale type of NVFP4 (pages
    "thinkingmachines/Inkling-2-Small", section Overview; "Thinking Machines releases Inkling 2 Small weights
    under Apache 2.0", section "NVFP4 and MXFP8 experts").
    """
    codes = np.asarray(codes).astype(np.int64)
    sign = np.where((codes >> 7) & 1, -1.0, 1.0)
    exp = (codes >> 3) & 15
    man = (codes & 7).astype(np.float64)
    normal = (1.0 + man / 8.0) * np.exp2(exp.astype(np.float64) - 7.0)
    sub = (man / 8.0) * 2.0 ** -6
    val = np.where(exp == 0, sub, normal)
    val = np.where((codes & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def e4m3_encode(v):
    """Round float values to E4M3FN, nearest-even, saturating to +-448.

    Works on the exact value of each input (float32 inputs are exact in
    float64).  Zero results are returned as +0 (code 0x00) whatever the
    sign of the input, the canonical zero of this library.

    Follows E4M3, the element type of the MXFP8 experts and the block-scale type of NVFP4 (pages
    "thinkingmachines/Inkling-2-Small", section Overview; "Thinking Machines releases Inkling 2 Small weights
    under Apache 2.0", section "NVFP4 and MXFP8 experts").
    """
    v = np.asarray(v, dtype=np.float64)
    if np.any(np.isnan(v)):
        raise ValueError("NaN input to e4m3_encode")
    sign = (v < 0).astype(np.int64)
    a = np.abs(v)
    mag = np.zeros(a.shape, dtype=np.int64)
    # subnormal range: value = m * 2^-9, m in 0..7 (m == 8 is the smallest normal)
    sub_mask = a < 2.0 ** -6
    m_sub = np.rint(a * 2.0 ** 9).astype(np.int64)      # exact scaling, RNE
    mag = np.where(sub_mask, m_sub, mag)                # code == m (8 -> 0x08 == 2^-6)
    # normal range
    with np.errstate(divide="ignore"):
        _, e2 = np.frexp(np.where(sub_mask, 1.0, a))    # a = f * 2^e2, f in [0.5, 1)
    E = e2 - 1                                          # a in [2^E, 2^(E+1))
    frac8 = np.where(sub_mask, 0.0, a / np.exp2(E.astype(np.float64)) - 1.0) * 8.0
    q = np.rint(frac8).astype(np.int64)                 # RNE on the exact fraction
    E = np.where(q == 8, E + 1, E)
    q = np.where(q == 8, 0, q)
    code_n = ((E + 7) << 3) | q
    mag = np.where(sub_mask, mag, code_n)
    mag = np.minimum(mag, 0x7E)                         # satfinite (also catches E > 8)
    mag = np.where(a >= E4M3_MAX, 0x7E, mag)
    out = np.where(mag == 0, 0, mag | (sign << 7))
    return out.astype(np.uint8)


# --------------------------------------------------------------------------
# E8M0
# --------------------------------------------------------------------------

def e8m0_decode(codes):
    """8-bit E8M0 codes -> float64 powers of two (NaN for 0xFF).

    Follows E8M0, the block-scale type of the MXFP8 experts (page "thinkingmachines/Inkling-2-Small", section
    Overview).
    """
    codes = np.asarray(codes).astype(np.int64)
    val = np.exp2(codes.astype(np.float64) - 127.0)
    return np.where(codes == 255, np.nan, val)


# --------------------------------------------------------------------------
# float32 helpers (one IEEE rounding per call, no fused multiply-add)
# --------------------------------------------------------------------------

def _f32(x):
    return np.asarray(x, dtype=np.float32)


def pairwise_tree_sum_f32(d):
    """Sum the last axis (length a power of two) by the fixed pairwise tree.

    Level by level: (d0+d1), (d2+d3), ... then ((d0+d1)+(d2+d3)), ...; every
    addition is a float32 addition.

    Follows the error sum of the 4-vs-6 pick (page "Thinking Machines releases Inkling 2 Small weights under
    Apache 2.0", section TL;DR); the pages fix no order, this tree is the order both implementations use.
    """
    s = _f32(d)
    while s.shape[-1] > 1:
        s = (s[..., 0::2] + s[..., 1::2]).astype(np.float32)
    return s[..., 0]


# --------------------------------------------------------------------------
# NVFP4 block quantizer with the 4-vs-6 scale pick
# --------------------------------------------------------------------------

NVFP4_BLOCK = 16
#: 6 (largest E2M1 magnitude) * 448 (largest E4M3 value)
NVFP4_TENSOR_DIVISOR = 2688.0


def nvfp4_tensor_scale(amax):
    """Second-level (tensor) scale s_g = amax / 2688 in float32; 1 when amax == 0.

    Follows the NVFP4 two-level scaling (page "Thinking Machines releases Inkling 2 Small weights under Apache
    2.0", section TL;DR); amax / (6 * 448) is the reading of the tensor scale.
    """
    amax = F32(amax)
    if amax == 0:
        return F32(1.0)
    return F32(amax / F32(NVFP4_TENSOR_DIVISOR))


def _nvfp4_candidate(x, a, s_g, c):
    """Quantize blocks x[..., 16] with the block maximum a mapped to c (4 or 6).

    Steps, all in float32 with one rounding each:
      e_c   = E4M3(a / (c * s_g))          block-scale code
      S_c   = dec(e_c) * s_g               effective block scale
      q_i   = sign(x_i) | E2M1(|x_i| / S_c)
      d_i   = x_i - dec(q_i) * S_c
      err_c = pairwise-tree sum of d_i * d_i
    If S_c is zero every code is zero and err_c is the tree sum of x_i * x_i.
    Returns (codes uint8[..., 16], scale code uint8[...], err float32[...]).

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section TL;DR: each
    block's maximum is mapped to 4 and to 6.
    """
    denom = (F32(c) * s_g).astype(np.float32)
    ratio = (a / denom).astype(np.float32)
    e_c = e4m3_encode(ratio)
    S_c = (_f32(e4m3_decode(e_c)) * s_g).astype(np.float32)
    zero = S_c == 0
    S_safe = np.where(zero, F32(1.0), S_c).astype(np.float32)[..., None]
    mag = e2m1_encode_magnitude((np.abs(x) / S_safe).astype(np.float32))
    neg = (x < 0) & (mag != 0)                       # a zero code is stored as +0
    codes = (mag | (neg.astype(np.int64) << 3))
    codes = np.where(zero[..., None], 0, codes).astype(np.uint8)
    recon = (_f32(e2m1_decode(codes)) * S_safe).astype(np.float32)
    d = (x - recon).astype(np.float32)
    d = np.where(zero[..., None], x, d).astype(np.float32)
    err = pairwise_tree_sum_f32((d * d).astype(np.float32))
    return codes, e_c, err


def nvfp4_quantize_blocks(x, s_g):
    """NVFP4 4-vs-6 quantization of float32 blocks x[..., 16].

    Returns (codes uint8[..., 16] with 4-bit E2M1 codes, scale codes uint8[...]
    in E4M3, chose_four bool[...]).  Candidate 4 is kept only when its error
    is strictly lower than candidate 6's (ties go to 6).

    Follows page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section TL;DR: the
    block is quantized both ways and the lower-error result is kept.
    """
    x = _f32(x)
    s_g = F32(s_g)
    assert x.shape[-1] == NVFP4_BLOCK
    if np.any(~np.isfinite(x)):
        raise ValueError("non-finite input to the NVFP4 quantizer")
    a = np.max(np.abs(x), axis=-1).astype(np.float32)
    c6, e6, err6 = _nvfp4_candidate(x, a, s_g, 6)
    c4, e4, err4 = _nvfp4_candidate(x, a, s_g, 4)
    four = err4 < err6
    codes = np.where(four[..., None], c4, c6).astype(np.uint8)
    scales = np.where(four, e4, e6).astype(np.uint8)
    return codes, scales, four


def nvfp4_quantize_rows(x, s_g):
    """Quantize a [rows, K] float32 matrix along K (K a multiple of 16).

    Returns (codes uint8[rows, K], scale codes uint8[rows, K/16]).

    Follows pages "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section TL;DR and
    "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    x = _f32(x)
    rows, K = x.shape
    assert K % NVFP4_BLOCK == 0
    codes, scales, _ = nvfp4_quantize_blocks(x.reshape(rows, K // NVFP4_BLOCK, NVFP4_BLOCK), s_g)
    return codes.reshape(rows, K), scales


def nvfp4_dequantize_rows(codes, scales, s_g):
    """Inverse of nvfp4_quantize_rows in float64: code * dec(scale) * s_g.

    Follows pages "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section TL;DR and
    "Thinking Machines releases Inkling 2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // NVFP4_BLOCK, NVFP4_BLOCK)
    v = v * e4m3_decode(scales)[..., None] * float(F32(s_g))
    return v.reshape(rows, K)


# --------------------------------------------------------------------------
# MXFP8 block quantizer
# --------------------------------------------------------------------------

MXFP8_BLOCK = 32
E4M3_EMAX = 8


def mxfp8_scale_exponent(amax):
    """OCP MX shared exponent: clamp(floor(log2 amax) - 8 + 127, 0, 254).

    floor(log2 amax) is taken exactly from the float32 exponent; amax == 0
    gives 0.  For float32 subnormal amax the result clamps to 0.

    Follows page "thinkingmachines/Inkling-2-Small", section Overview (MXFP8 experts in layers 40-47); the
    shared exponent as the OCP MX v1.0 rule.
    """
    amax = np.asarray(amax, dtype=np.float64)
    with np.errstate(divide="ignore"):
        _, e2 = np.frexp(np.where(amax > 0, amax, 1.0))
    fl = e2 - 1                                  # floor(log2 amax) for amax > 0
    e = np.clip(fl - E4M3_EMAX + 127, 0, 254)
    return np.where(amax > 0, e, 0).astype(np.uint8)


def mxfp8_quantize_blocks(x):
    """MXFP8 quantization of float32 blocks x[..., 32].

    q_i = E4M3(x_i * 2^(127 - e)); multiplying by a power of two is exact
    here (see mxfp8_scale_exponent), and values that land in (448, 512)
    saturate to 448.  Returns (codes uint8[..., 32], scale codes uint8[...]).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    x = _f32(x)
    assert x.shape[-1] == MXFP8_BLOCK
    if np.any(~np.isfinite(x)):
        raise ValueError("non-finite input to the MXFP8 quantizer")
    a = np.max(np.abs(x), axis=-1)
    e = mxfp8_scale_exponent(a)
    scaled = x.astype(np.float64) * np.exp2(127.0 - e.astype(np.float64))[..., None]
    codes = e4m3_encode(scaled)
    return codes, e


def mxfp8_quantize_rows(x):
    """Quantize a [rows, K] float32 matrix along K (K a multiple of 32).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    x = _f32(x)
    rows, K = x.shape
    assert K % MXFP8_BLOCK == 0
    codes, scales = mxfp8_quantize_blocks(x.reshape(rows, K // MXFP8_BLOCK, MXFP8_BLOCK))
    return codes.reshape(rows, K), scales


def mxfp8_dequantize_rows(codes, scales):
    """Inverse of mxfp8_quantize_rows in float64: code * 2^(e - 127).

    Follows pages "thinkingmachines/Inkling-2-Small", section Overview and "Thinking Machines releases Inkling
    2 Small weights under Apache 2.0", section "NVFP4 and MXFP8 experts".
    """
    rows, K = codes.shape
    v = e4m3_decode(codes).reshape(rows, K // MXFP8_BLOCK, MXFP8_BLOCK)
    v = v * e8m0_decode(scales)[..., None]
    return v.reshape(rows, K)


# --------------------------------------------------------------------------
# bfloat16 rounding (for the layer output)
# --------------------------------------------------------------------------

def bf16_round(v):
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    Direct rounding of the exact value to 8 significant bits; magnitudes
    below the smallest normal bfloat16 round on the subnormal grid 2^-133.

    Follows the reading that the layer's input x and output y are bf16 (the pages state no activation type);
    rounding to nearest, ties to even.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        _, e2 = np.frexp(np.where(a > 0, a, 1.0))
    E = np.maximum(e2 - 1, -126)                # exponent of the leading bit
    ulp = np.exp2(E.astype(np.float64) - 7.0)   # 8 significant bits
    r = np.rint(a / ulp) * ulp
    r = np.where(a > 0, r, 0.0)
    return np.copysign(r, v)
