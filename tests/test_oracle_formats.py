"""Pins of the oracle's number formats and block quantizers (CPU only).

Each check compares the oracle with something other than itself: the
ml_dtypes casts (a library implementation of the OCP formats), exact
rational arithmetic (fractions), brute force over every code, or the
hand-worked examples in tests/golden/ (page "Thinking Machines releases
Inkling 2 Small weights under Apache 2.0", section TL;DR).
"""

import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from oracle import formats as fm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
             Fraction(3), Fraction(4), Fraction(6)]


# ---------------------------------------------------------------- decoders

def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(fm.e2m1_decode(codes), ref)


def test_e4m3_decode_matches_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = fm.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert fm.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert fm.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9


def test_e8m0_decode_matches_ml_dtypes():
    codes = np.arange(255, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    np.testing.assert_array_equal(fm.e8m0_decode(codes), ref)
    assert np.isnan(fm.e8m0_decode(np.array([255]))[0])


# ---------------------------------------------------------------- encoders

def _around(points):
    """float32 points plus their float32 neighbours on both sides."""
    p = np.asarray(points, dtype=np.float32)
    return np.concatenate([p, np.nextafter(p, np.float32(np.inf)),
                           np.nextafter(p, np.float32(-np.inf))])


def test_e2m1_encode_matches_ml_dtypes_rne():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = np.concatenate([_around(mids + list(fm.E2M1_MAGNITUDES[1:])),
                           np.random.default_rng(0).uniform(0, 6, 20000).astype(np.float32)])
    vals = vals[vals >= 0]
    ref = vals.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.asarray(fm.E2M1_MAGNITUDES)[fm.e2m1_encode_magnitude(vals)]
    np.testing.assert_array_equal(got, ref)
    # saturation above 6
    assert fm.e2m1_encode_magnitude(np.array([7.0, 100.0, 5.0000001])).tolist() == [7, 7, 7]


def test_e4m3_encode_matches_ml_dtypes_on_clipped_values():
    rng = np.random.default_rng(1)
    mags = np.exp2(rng.uniform(-14, 10, 50000)).astype(np.float32)
    codes_all = np.arange(0x7F, dtype=np.uint8)
    reps = codes_all.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = ((reps[1:] + reps[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([mags, _around(mids), _around(reps.astype(np.float32)),
                           np.array([448, 449, 464, 465, 1e6, 0.0], dtype=np.float32)])
    vals = np.concatenate([vals, -vals])
    clipped = np.clip(vals, -448, 448)
    ref = clipped.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = fm.e4m3_decode(fm.e4m3_encode(vals))
    np.testing.assert_array_equal(got, ref)
    # canonical +0 for every zero result
    assert fm.e4m3_encode(np.array([-0.0, -1e-30], dtype=np.float32)).tolist() == [0, 0]


# ---------------------------------------------------------------- NVFP4 4-vs-6

def _exact_e4m3_code(q):
    """E4M3 code nearest (ties to even) to the exact rational q >= 0, saturating."""
    best = None
    for code in range(0x7F):
        v = Fraction(fm.e4m3_decode(np.array([code]))[0])
        d = abs(v - q)
        key = (d, code & 1)              # on a tie the even mantissa wins
        if best is None or key < best[0]:
            best = (key, code)
    return best[1]


def _exact_block_error(x, S):
    """Exact squared error of the E2M1 quantization of block x at scale S > 0.

    Each element takes the magnitude that minimizes |x| - m*S (ties to the
    even code, i.e. the magnitude whose mantissa bit is 0).
    """
    err = Fraction(0)
    codes = []
    for xi in x:
        a = abs(Fraction(float(xi)))
        best = None
        for c, m in enumerate(E2M1_MAGS):
            key = (abs(a - m * S), c & 1)
            if best is None or key < best[0]:
                best = (key, c, m)
        _, c, m = best
        r = m * S
        err += (a - r) ** 2
        codes.append(c | (8 if (xi < 0 and c != 0) else 0))
    return err, codes


def _random_blocks(n, seed):
    rng = np.random.default_rng(seed)
    kinds = []
    for i in range(n):
        k = i % 4
        if k == 0:
            b = rng.standard_normal(16)
        elif k == 1:                       # heavy tail
            b = rng.standard_t(2, 16)
        elif k == 2:                       # one outlier
            b = rng.standard_normal(16) * 0.1
            b[rng.integers(16)] = rng.uniform(1, 4)
        else:                              # values on the E2M1 grid times a scale
            b = rng.choice([0, .5, 1, 1.5, 2, 3, 4, 6], 16) * rng.choice([-1, 1], 16) * rng.uniform(0.2, 3)
        kinds.append(b)
    return np.asarray(kinds, dtype=np.float32)


@pytest.mark.parametrize("s_g", [1.0, 0.0123, 3.7e-3, 2.0 ** -7])
def test_nvfp4_choice_against_exact_rational_search(s_g):
    s_g = np.float32(s_g)
    blocks = _random_blocks(160, seed=int(s_g * 1e6) + 7)
    codes, scales, four = fm.nvfp4_quantize_blocks(blocks, s_g)
    sg = Fraction(float(s_g))
    for b, c, s, f4 in zip(blocks, codes, scales, four):
        a = max(abs(Fraction(float(v))) for v in b)
        cand = {}
        for c_map in (4, 6):
            e = _exact_e4m3_code(a / (c_map * sg))
            S = Fraction(fm.e4m3_decode(np.array([e]))[0]) * sg
            if S == 0:
                err, cc = sum(Fraction(float(v)) ** 2 for v in b), [0] * 16
            else:
                err, cc = _exact_block_error(b, S)
            cand[c_map] = (e, S, err, cc)
        # the chosen scale is one of the two candidates
        assert int(s) in (cand[4][0], cand[6][0])
        chosen = cand[4] if f4 else cand[6]
        assert int(s) == chosen[0]
        # codes are the nearest E2M1 values at the chosen scale
        if chosen[1] != 0:
            assert [int(v) for v in c] == chosen[3]
        # the choice agrees with the exact squared errors (ties to 6) unless the
        # two errors are within float32 rounding of each other
        e4, e6 = cand[4][2], cand[6][2]
        exact_four = e4 < e6
        if exact_four != bool(f4):
            assert abs(e4 - e6) <= Fraction(1, 2 ** 18) * max(e4, e6, Fraction(1, 10 ** 30))
        # never worse than plain NVFP4 (map to 6 only), up to float32 rounding
        assert chosen[2] <= e6 * (1 + Fraction(1, 2 ** 18))


def test_nvfp4_against_brute_force_over_all_scales():
    """The best of all 127 E4M3 scales is never better than the 4-vs-6 pick by
    more than the search space allows, and the pick is the best of its two
    candidates; on blocks built from E2M1 values at an E4M3 scale the pick is
    exact (error 0)."""
    rng = np.random.default_rng(5)
    s_g = np.float32(1.0)
    for _ in range(40):
        scale = fm.e4m3_decode(np.array([rng.integers(0x20, 0x50)]))[0]
        mags = rng.choice([0, .5, 1, 1.5, 2, 3, 4, 6], 16)
        mags[0] = 6.0
        b = (mags * rng.choice([-1, 1], 16) * scale).astype(np.float32)
        codes, scales, four = fm.nvfp4_quantize_blocks(b[None], s_g)
        S = Fraction(fm.e4m3_decode(scales)[0])
        err, _ = _exact_block_error(b, S)
        assert err == 0
    # brute force over every scale code on random blocks
    for b in _random_blocks(24, seed=11):
        codes, scales, four = fm.nvfp4_quantize_blocks(b[None], s_g)
        S_pick = Fraction(fm.e4m3_decode(scales)[0])
        err_pick = _exact_block_error(b, S_pick)[0] if S_pick else sum(Fraction(float(v)) ** 2 for v in b)
        all_errs = []
        for code in range(1, 0x7F):
            S = Fraction(fm.e4m3_decode(np.array([code]))[0])
            all_errs.append(_exact_block_error(b, S)[0])
        assert min(all_errs) <= err_pick


def test_nvfp4_tie_goes_to_six():
    # 3.0 is exact for both candidates (6 * 0.5 and 4 * 0.75): a tie at error 0
    b = np.zeros((1, 16), dtype=np.float32)
    b[0, 0] = 3.0
    codes, scales, four = fm.nvfp4_quantize_blocks(b, np.float32(1.0))
    assert not four[0]
    assert fm.e4m3_decode(scales)[0] == 0.5 and codes[0, 0] == 7


def test_nvfp4_saturated_four_candidate_is_still_scored():
    # block max 2400 with s_g = 1: a/4 = 600 saturates to 448, a/6 = 400 does not
    b = np.zeros((1, 16), dtype=np.float32)
    b[0, 0] = 2400.0
    b[0, 1] = 1700.0
    codes, scales, four = fm.nvfp4_quantize_blocks(b, np.float32(1.0))
    e4 = fm.e4m3_encode(np.float32(600.0))
    assert e4 == 0x7E
    # candidate 4 at scale 448: 2400/448 = 5.36 -> 6 (2688), 1700/448 = 3.79 -> 4 (1792)
    # candidate 6 at scale 400: 2400/400 = 6 (2400), 1700/400 = 4.25 -> 4 (1600)
    # errors: c4 = 288^2 + 92^2, c6 = 0 + 100^2 -> 6 wins
    assert not four[0]


def test_nvfp4_golden_examples():
    with open(os.path.join(GOLDEN, "nvfp4_4v6_examples.json")) as f:
        gold = json.load(f)
    for ex in gold["examples"]:
        b = np.asarray(ex["block"], dtype=np.float32)[None]
        codes, scales, four = fm.nvfp4_quantize_blocks(b, np.float32(gold["s_g"]))
        assert int(scales[0]) == ex["scale_code"]
        assert fm.e4m3_decode(scales)[0] == ex["scale_value"]
        assert [int(c) for c in codes[0]] == ex["codes"]
        assert bool(four[0]) == ex["chose_four"]


def test_nvfp4_tensor_scale():
    assert fm.nvfp4_tensor_scale(np.float32(2688.0)) == np.float32(1.0)
    assert fm.nvfp4_tensor_scale(np.float32(0.0)) == np.float32(1.0)
    # the largest element of a tensor maps onto the top of the two-level range
    x = np.random.default_rng(3).standard_normal((8, 64)).astype(np.float32)
    s = fm.nvfp4_tensor_scale(np.max(np.abs(x)))
    codes, sf = fm.nvfp4_quantize_rows(x, s)
    assert fm.e4m3_decode(sf).max() <= 448.0
    deq = fm.nvfp4_dequantize_rows(codes, sf, s)
    assert np.max(np.abs(deq - x)) <= np.max(np.abs(x)) / 6 * 1.01


def test_pairwise_tree_order():
    # the tree sum differs from a left-to-right sum on this input
    d = np.array([1e8, 1, -1e8, 1] + [0] * 12, dtype=np.float32)
    assert fm.pairwise_tree_sum_f32(d) == np.float32((np.float32(1e8 + 1) + np.float32(-1e8 + 1)))


# ---------------------------------------------------------------- MXFP8

def test_mxfp8_scale_closed_form():
    import math
    rng = np.random.default_rng(4)
    amax = np.exp2(rng.uniform(-130, 120, 4000)).astype(np.float32)
    amax = amax[amax > 0]
    got = fm.mxfp8_scale_exponent(amax)
    for a, e in zip(amax[:500], got[:500]):
        m, ex = math.frexp(float(a))
        assert e == min(max(ex - 1 - 8 + 127, 0), 254)
    assert fm.mxfp8_scale_exponent(np.array([0.0]))[0] == 0
    assert fm.mxfp8_scale_exponent(np.array([1.0]))[0] == 119     # 2^0 -> 127 - 8
    assert fm.mxfp8_scale_exponent(np.array([448.0]))[0] == 127


def test_mxfp8_codes_match_library_cast():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((300, 32)) * np.exp2(rng.uniform(-20, 20, (300, 1)))).astype(np.float32)
    x[0] = 0.0
    x[1, :] = 0.0
    x[1, 3] = 500.0 * 2.0 ** -10          # lands in (448, 512) after scaling
    codes, e = fm.mxfp8_quantize_blocks(x)
    scaled = x.astype(np.float64) * np.exp2(127.0 - e.astype(np.float64))[:, None]
    ref = np.clip(scaled, -448, 448).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(fm.e4m3_decode(codes), ref)
    assert fm.e4m3_decode(codes[1, 3:4])[0] == 448.0
    # dequantized error bounded by half an E4M3 ulp at the block scale
    deq = fm.mxfp8_dequantize_rows(codes, e[:, None])
    scale = fm.e8m0_decode(e)[:, None]
    sat = np.abs(x) > 448.0 * scale            # OCP rule: block maxima in (448, 512) saturate
    np.testing.assert_array_equal(np.abs(deq[sat]), (448.0 * np.broadcast_to(scale, x.shape))[sat])
    ok = ~sat
    bound = np.abs(x) * 2.0 ** -4 + scale * 2.0 ** -10      # half an E4M3 ulp
    assert np.all((np.abs(deq - x) <= bound)[ok])


def test_bf16_round_matches_torch():
    import torch
    v = np.random.default_rng(8).standard_normal(20000) * 10
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = fm.bf16_round(v.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def _quotients(h, S):
    """(definition, fast) float32 quotients |h| / S and |h| * RN(1/S)."""
    ax, Sv = np.abs(h).astype(np.float32), S.astype(np.float32)
    q_def = (ax / Sv).astype(np.float32)
    q_fast = (ax * (np.float32(1.0) / Sv).astype(np.float32)).astype(np.float32)
    return ax, Sv, q_def, q_fast


def test_fast_h_quotient_differs_only_next_to_a_midpoint():
    """Bound behind the 1e-3 bar on intermediate codes: the GEMM epilogue
    rounds |h| * RN(1/S) where the definition (and the oracle) rounds |h| / S.
    Two float32 roundings put the fast quotient within a relative 2^-23 of
    the exact one, so the E2M1 code can differ only where |h| / S lies that
    close to a rounding midpoint.  On SwiGLU-shaped blocks at the static
    scale (both candidates' block scales) no code differs; on values placed
    a few ulps from a midpoint some do, and every one of them is next to it."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rng = np.random.default_rng(17)
    # SwiGLU-shaped blocks
    n = 200000
    g = rng.standard_normal((n, 16)) * 2.0
    u = rng.standard_normal((n, 16)) * 2.0
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    s_g = np.float32(24 / 2688)
    a = np.max(np.abs(h), axis=1).astype(np.float32)
    for c in (6, 4):
        e = fm.e4m3_encode((a / (np.float32(c) * s_g).astype(np.float32)).astype(np.float32))
        S = (fm.e4m3_decode(e).astype(np.float32) * s_g).astype(np.float32)
        ok = S > 0
        ax, Sv, q_def, q_fast = _quotients(h[ok], S[ok][:, None])
        exact = ax.astype(np.float64) / Sv.astype(np.float64)
        assert np.all(np.abs(q_fast - exact) <= 2.0 ** -23 * exact + 1e-45)
        differ = fm.e2m1_encode_magnitude(q_def) != fm.e2m1_encode_magnitude(q_fast)
        assert differ.sum() <= 1e-4 * differ.size
    # values a few float32 ulps from a midpoint, at random block scales
    codes = rng.integers(0x08, 0x7F, 4000)
    S = (fm.e4m3_decode(codes).astype(np.float32) * s_g).astype(np.float32)[:, None]
    offs = np.arange(-4, 5) * 2.0 ** -23
    hv = (mids[None, :, None] * (1 + offs)[None, None, :] * S[:, :, None].astype(np.float64)).astype(np.float32)
    hv = hv.reshape(len(codes), -1)
    ax, Sv, q_def, q_fast = _quotients(hv, S)
    differ = fm.e2m1_encode_magnitude(q_def) != fm.e2m1_encode_magnitude(q_fast)
    assert differ.any()                          # the bound is reached: the bar cannot be zero
    exact = (ax.astype(np.float64) / Sv.astype(np.float64))[differ]
    near = np.min(np.abs(exact[:, None] / mids[None, :] - 1.0), axis=1)
    assert np.all(near <= 2.0 ** -22), near.max()

def _e2m1_value(code):
    return np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)[code]


def test_fast_h_error_sum_changes_the_pick_only_on_near_ties():
    """Second departure behind the 1e-3 bar on intermediate codes: the GEMM
    epilogue accumulates a candidate's squared error with fused multiply-adds
    (d = fma(-v, S, |h|), then e = fma(d, d, e) over even and odd elements,
    the two sums added) where the definition rounds every product and
    difference and sums pairwise.  Emulated here on SwiGLU-shaped blocks (the
    fused operations as one float64 evaluation rounded to float32; the
    element codes from the same fast quotient on both sides, so only the sum
    differs): the 4-vs-6 pick differs on a tiny fraction of blocks, and only
    where the two candidates' errors nearly tie."""
    rng = np.random.default_rng(29)
    n = 200000
    g = rng.standard_normal((n, 16)) * 2.0
    u = rng.standard_normal((n, 16)) * 2.0
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    s_g = np.float32(24 / 2688)
    a = np.max(np.abs(h), axis=1).astype(np.float32)
    f32 = np.float32
    err_def, err_fast = {}, {}
    for c in (6, 4):
        e = fm.e4m3_encode((a / (f32(c) * s_g).astype(f32)).astype(f32))
        S = (fm.e4m3_decode(e).astype(f32) * s_g).astype(f32)[:, None]
        ax = np.abs(h)
        q = (ax * (f32(1.0) / S).astype(f32)).astype(f32)
        v = _e2m1_value(fm.e2m1_encode_magnitude(q))
        # definition: RN(v S), RN(|h| - .), RN(d d), pairwise tree
        d = (ax - (v * S).astype(f32)).astype(f32)
        t = (d * d).astype(f32)
        while t.shape[1] > 1:
            t = (t[:, 0::2] + t[:, 1::2]).astype(f32)
        err_def[c] = t[:, 0]
        # fused: d = RN(|h| - v S), e = RN(d d + e), even / odd running sums
        df = (ax.astype(np.float64) - v.astype(np.float64) * S.astype(np.float64)).astype(f32)
        e0 = np.zeros(n, dtype=f32)
        e1 = np.zeros(n, dtype=f32)
        for i in range(0, 16, 2):
            e0 = (df[:, i].astype(np.float64) ** 2 + e0.astype(np.float64)).astype(f32)
            e1 = (df[:, i + 1].astype(np.float64) ** 2 + e1.astype(np.float64)).astype(f32)
        err_fast[c] = (e0 + e1).astype(f32)
    ok = a > 0
    pick_def = (err_def[4] < err_def[6])[ok]
    pick_fast = (err_fast[4] < err_fast[6])[ok]
    differ = pick_def != pick_fast
    assert differ.sum() <= 1e-4 * differ.size, differ.sum()
    e4, e6 = err_def[4][ok][differ].astype(np.float64), err_def[6][ok][differ].astype(np.float64)
    assert np.all(np.abs(e4 - e6) <= 2.0 ** -18 * np.maximum(e4, e6)), np.max(np.abs(e4 - e6) / np.maximum(e4, e6))
