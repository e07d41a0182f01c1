"""Pins of the oracle's routing, permutation, FFN and combine (CPU only).

Routing follows the pages "thinkingmachines/Inkling-2-Small" (Overview) and
"Thinking Machines releases Inkling 2 Small weights under Apache 2.0"
("NVFP4 and MXFP8 experts"): top-k of E routed experts, no shared expert.
The checks compare with numpy's stable argsort and bincount (library
routines), math.exp, a dense FFN written out directly, and a per-token loop.
"""

import math

import numpy as np
import pytest

from oracle import formats as fm
from oracle import moe
from oracle import route as rt
from fp8_moe_expert_top_b200 import inputs


# ---------------------------------------------------------------- exp_own

def test_exp_own_accuracy_against_math_exp():
    x = np.concatenate([np.linspace(-80, 0, 200001), -np.exp2(np.linspace(-30, 6, 2000))]).astype(np.float32)
    got = rt.exp_own(x).astype(np.float64)
    ref = np.array([math.exp(float(v)) for v in x])
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 3 * 2.0 ** -24, rel.max()
    assert rt.exp_own(np.float32(0.0)) == np.float32(1.0)
    assert rt.exp_own(np.float32(-80.5)) == 0.0


# ---------------------------------------------------------------- router scores

def _f32_nearest(q):
    """The float32 nearest to the rational q, ties to the even significand
    (decided exactly with fractions)."""
    from fractions import Fraction
    f = np.float32(float(q))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - q), int(np.float32(c).view(np.uint32)) & 1))


def _bf16_values(rng, shape, scale=1.0):
    import torch
    v = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16)
    return v.float().numpy()


@pytest.mark.parametrize("spread", [False, True])
def test_router_logits_against_exact_rational_sums(spread):
    """Every score is the float32 rounding of the exact sum of bf16 products
    (also when the products span many binades, so that a float32 running sum
    would drop low bits)."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    T, E, H = 8, 16, 256
    x = _bf16_values(rng, (T, H))
    if spread:
        x = _bf16_values(rng, (T, H)) * np.exp2(rng.integers(-12, 13, (T, H))).astype(np.float32)
    w = _bf16_values(rng, (E, H), 1.0 / 16)
    got = rt.router_logits(x, w)
    assert got.dtype == np.float32 and got.shape == (T, E)
    xf = [[Fraction(float(v)) for v in row] for row in x]
    wf = [[Fraction(float(v)) for v in row] for row in w]
    for t in range(T):
        for e in range(E):
            q = sum(a * b for a, b in zip(xf[t], wf[e]))
            assert got[t, e] == _f32_nearest(q), (t, e, got[t, e], float(q))


def test_router_logits_of_one_hot_rows():
    """A token that is a scaled unit vector scores each expert with that
    column of the router weights, exactly."""
    rng = np.random.default_rng(12)
    w = _bf16_values(rng, (5, 16))
    x = np.zeros((3, 16), dtype=np.float32)
    x[0, 3], x[1, 15], x[2, 0] = 1.0, -2.0, 0.5
    got = rt.router_logits(x, w)
    np.testing.assert_array_equal(got[0], w[:, 3])
    np.testing.assert_array_equal(got[1], -2.0 * w[:, 15])
    np.testing.assert_array_equal(got[2], 0.5 * w[:, 0])


def test_router_route_equal_router_rows_tie_to_lower_index():
    """Two experts with the same router row score the same on every token;
    whenever both are selected the lower index comes first."""
    rng = np.random.default_rng(13)
    w = _bf16_values(rng, (12, 32))
    w[9] = w[2]
    x = _bf16_values(rng, (400, 32))
    r = rt.router_route(x, w, 4, 12)
    both = 0
    for row in r["topk_ids"].tolist():
        if 2 in row and 9 in row:
            both += 1
            assert row.index(2) + 1 == row.index(9)
        assert 9 not in row or 2 in row
    assert both > 0


# ---------------------------------------------------------------- top-k

@pytest.mark.parametrize("ties", [False, True])
def test_topk_matches_stable_argsort(ties):
    T, E, k = 300, 384, 8
    if ties:
        lg = inputs.make_logits_with_ties(T, E, seed=3).numpy()
    else:
        lg = np.random.default_rng(2).standard_normal((T, E)).astype(np.float32)
    ids = rt.topk_select(lg, k)
    ref = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(ids, ref)


def test_topk_signed_zero_ties_to_lower_index():
    lg = np.full((1, 6), -1.0, dtype=np.float32)
    lg[0, 4] = 0.0
    lg[0, 1] = -0.0
    ids = rt.topk_select(lg, 2)
    assert ids.tolist() == [[1, 4]]


def test_softmax_weights():
    lg = np.random.default_rng(4).standard_normal((50, 16)).astype(np.float32)
    ids = rt.topk_select(lg, 1)
    assert np.all(rt.topk_softmax(lg, ids) == np.float32(1.0))
    ids = rt.topk_select(lg, 4)
    w = rt.topk_softmax(lg, ids)
    sel = np.take_along_axis(lg.astype(np.float64), ids.astype(np.int64), axis=1)
    ref = np.exp(sel - sel[:, :1])
    ref /= ref.sum(1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=4e-7)
    assert np.all(np.diff(w, axis=1) <= 0)             # rank order


def test_softmax_weights_of_large_logits():
    """Softmax is defined for any finite logits: rows offset far from zero
    (where exp of a raw logit overflows float32) still give the float64 weights."""
    rng = np.random.default_rng(12)
    lg = (rng.standard_normal((40, 16)) * 3 + rng.choice([-300.0, 150.0, 1000.0], (40, 1))).astype(np.float32)
    ids = rt.topk_select(lg, 8)
    w = rt.topk_softmax(lg, ids)
    sel = np.take_along_axis(lg.astype(np.float64), ids.astype(np.int64), axis=1)
    ref = np.exp(sel - sel.max(1, keepdims=True))
    ref /= ref.sum(1, keepdims=True)
    assert np.all(np.isfinite(w))
    np.testing.assert_allclose(w, ref, rtol=4e-7, atol=1e-30)


# ---------------------------------------------------------------- slot sort

def test_sort_slots_matches_library_sort():
    rng = np.random.default_rng(5)
    T, E, k = 200, 24, 3
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, 5] += 3.0                                     # one hot expert
    lg[:, 7] -= 50.0                                    # one cold expert (no slots)
    ids = rt.topk_select(lg, k)
    counts, offsets, sorted_slots, slot_to_row = rt.sort_slots(ids, E)
    flat = ids.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    assert counts[7] == 0
    seg = np.diff(offsets)
    assert np.all(offsets % 128 == 0)
    np.testing.assert_array_equal(seg, (counts + 127) // 128 * 128)
    # valid rows in (expert, token) order == a stable sort of the slots by expert
    order = np.argsort(flat, kind="stable")
    valid = sorted_slots[sorted_slots >= 0]
    np.testing.assert_array_equal(valid, order)
    # inverse map and padding
    assert np.all(slot_to_row[sorted_slots[sorted_slots >= 0]] == np.nonzero(sorted_slots >= 0)[0])
    for e in range(E):
        lo = offsets[e]
        assert np.all(sorted_slots[lo + counts[e]:offsets[e + 1]] == -1)
        assert np.all(flat[sorted_slots[lo:lo + counts[e]]] == e)


def test_combine_of_passthrough_is_identity():
    """Permute x by the slot sort, combine with k=1 and w=1: y == x exactly."""
    rng = np.random.default_rng(6)
    T, E, H = 40, 6, 32
    x = fm.bf16_round(rng.standard_normal((T, H)))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    r = rt.route(lg, 1, E)
    rows = np.zeros((r["sorted_slots"].shape[0], H))
    valid = r["sorted_slots"] >= 0
    rows[valid] = x[r["sorted_slots"][valid]]
    y = moe.combine(rows, r["topk_w"], r["slot_to_row"])
    np.testing.assert_array_equal(y, x)


# ---------------------------------------------------------------- the layer

def _small_case(fmt, T=24, H=64, I=32, E=4, k=2, seed=7):
    rng = np.random.default_rng(seed)
    x = fm.bf16_round(rng.standard_normal((T, H))).astype(np.float32)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    experts = {}
    raw = {}
    for e in range(E):
        wg = (rng.standard_normal((I, H)) / math.sqrt(H)).astype(np.float32)
        wu = (rng.standard_normal((I, H)) / math.sqrt(H)).astype(np.float32)
        wd = (rng.standard_normal((H, I)) / math.sqrt(I)).astype(np.float32)
        raw[e] = (wg, wu, wd)
        experts[e] = moe.quantize_expert(wg, wu, wd, fmt)
    return x, lg, experts, raw


@pytest.mark.parametrize("fmt", [moe.NVFP4, moe.MXFP8])
def test_one_expert_layer_equals_dense_ffn(fmt):
    """E = 1, k = 1: the routed layer is exactly the dense FFN of that expert."""
    x, lg, experts, raw = _small_case(fmt, T=16, H=64, I=32, E=1, k=1)
    s_x, s_h = np.float32(8 / 2688), np.float32(24 / 2688)
    res = moe.forward(x, lg, experts, 1, fmt, s_x, s_h)
    # dense FFN written out: quantize x, dequantize, GEMM, SwiGLU, requantize, GEMM
    if fmt == moe.NVFP4:
        xc, xs = fm.nvfp4_quantize_rows(x, s_x)
        xd = fm.nvfp4_dequantize_rows(xc, xs, s_x)
    else:
        xc, xs = fm.mxfp8_quantize_rows(x)
        xd = fm.mxfp8_dequantize_rows(xc, xs)
    q = experts[0]
    deq = {}
    for m, (c, s, ts) in q.items():
        deq[m] = (fm.nvfp4_dequantize_rows(c, s, ts) if fmt == moe.NVFP4
                  else fm.mxfp8_dequantize_rows(c, s))
    g = xd @ deq["gate"].T
    u = xd @ deq["up"].T
    h = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
    if fmt == moe.NVFP4:
        hc, hs = fm.nvfp4_quantize_rows(h, s_h)
        hd = fm.nvfp4_dequantize_rows(hc, hs, s_h)
    else:
        hc, hs = fm.mxfp8_quantize_rows(h)
        hd = fm.mxfp8_dequantize_rows(hc, hs)
    y = fm.bf16_round(hd @ deq["down"].T)
    np.testing.assert_array_equal(res["y"], y)
    np.testing.assert_array_equal(res["gate"][:16], g)
    # and the quantized FFN is a close approximation of the float FFN
    wg, wu, wd = raw[0]
    gf = x.astype(np.float64) @ wg.T
    uf = x.astype(np.float64) @ wu.T
    yf = (gf / (1 + np.exp(-gf)) * uf) @ wd.T
    rel = np.linalg.norm(res["y"] - yf) / np.linalg.norm(yf)
    assert rel < (0.25 if fmt == moe.NVFP4 else 0.08), rel


@pytest.mark.parametrize("fmt", [moe.NVFP4, moe.MXFP8])
def test_layer_equals_per_token_loop(fmt):
    """The permuted-matrix forward equals a token-by-token evaluation."""
    x, lg, experts, _ = _small_case(fmt, T=24, E=5, k=2, seed=9)
    s_x, s_h = np.float32(8 / 2688), np.float32(24 / 2688)
    res = moe.forward(x, lg, experts, 2, fmt, s_x, s_h)
    ref = moe.forward_tokens(x, lg, experts, 2, fmt, s_x, s_h)
    np.testing.assert_array_equal(res["topk_ids"], ref["topk_ids"])
    np.testing.assert_array_equal(res["topk_w"], ref["topk_w"])
    np.testing.assert_allclose(res["y"], ref["y"], rtol=2 ** -7, atol=1e-6)
    diff = np.mean(res["y"] != ref["y"])
    assert diff < 0.02       # only float64 summation order differs, then bf16 rounding


def test_weight_tensor_scale_maps_largest_magnitude_to_top_of_range():
    """NVFP4 weights: the element of largest magnitude lands on the top of the
    two-level range (code +-6 at block scale 448) and is reproduced, whatever
    its sign; every other element stays inside the range."""
    rng = np.random.default_rng(13)
    for sign in (-1.0, 1.0):
        w = (rng.standard_normal((32, 64)) * 0.02).astype(np.float32)
        w[5, 17] = sign * 0.5                           # the extreme element, either sign
        q = moe.quantize_expert(w, w, w.T.copy(), moe.NVFP4)
        codes, sf, s_g = q["gate"]
        deq = fm.nvfp4_dequantize_rows(codes, sf, s_g)
        assert sf[5, 17 // 16] == 0x7E
        assert codes[5, 17] == (15 if sign < 0 else 7)
        assert abs(deq[5, 17] - w[5, 17]) <= 2.0 ** -22 * 0.5
        assert np.max(np.abs(deq)) <= 0.5 * (1 + 2.0 ** -22)


def test_expert_ffn_gemms_against_exact_sums():
    """Brute force on a tiny expert: with operands on the E2M1 grid times
    powers of two (so every product and partial sum is exact in float64) the
    oracle's gate and up outputs equal the exact rational sums element by
    element, and its down output is within float64 rounding of the exact sum
    over its own dequantized intermediate."""
    from fractions import Fraction
    rng = np.random.default_rng(21)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    m, H, I = 3, 32, 32

    def rand(shape):
        return rng.choice(grid, shape) * rng.choice([-1, 1], shape) * np.exp2(rng.integers(-3, 4, shape))

    a, wg, wu, wd = rand((m, H)), rand((I, H)), rand((I, H)), rand((H, I))

    def exact(A, W):                       # A [m, K] times W [n, K] transposed, in rationals
        return [[sum(Fraction(float(A[i, c])) * Fraction(float(W[j, c])) for c in range(A.shape[1]))
                 for j in range(W.shape[0])] for i in range(A.shape[0])]

    f = moe.expert_ffn(a, dict(gate=wg, up=wu, down=wd), moe.MXFP8, None)
    assert f["gate"].tolist() == [[float(v) for v in row] for row in exact(a, wg)]
    assert f["up"].tolist() == [[float(v) for v in row] for row in exact(a, wu)]
    h_deq = fm.mxfp8_dequantize_rows(f["h_codes"], f["h_sf"])
    o = exact(h_deq, wd)
    bound = I * 2.0 ** -52 * (np.abs(h_deq) @ np.abs(wd).T)
    for i in range(m):
        for j in range(H):
            assert abs(Fraction(float(f["out"][i, j])) - o[i][j]) <= Fraction(float(bound[i, j]))


def test_swiglu_closed_form():
    g = np.array([0.0, 1.0, -1.0, 10.0, -30.0])
    u = np.array([2.0, 3.0, 1.0, 1.0, 1.0])
    ref = np.array([0.0, 3.0 / (1 + math.exp(-1.0)), -1.0 / (1 + math.e), 10.0 / (1 + math.exp(-10.0)),
                    -30.0 / (1 + math.exp(30.0))])
    np.testing.assert_allclose(moe.swiglu(g, u), ref, rtol=1e-15)


@pytest.mark.parametrize("fmt", [moe.NVFP4, moe.MXFP8])
def test_degenerate_batches(fmt):
    """An empty batch gives an empty output and no rows; k = E sends every
    token to every expert (weights a softmax over all E logits, every segment
    holding all T tokens in order); a single token equals its per-token
    evaluation."""
    x, lg, experts, _ = _small_case(fmt, T=5, E=3, k=3, seed=11)
    s_x, s_h = np.float32(8 / 2688), np.float32(24 / 2688)
    empty = moe.forward(x[:0], lg[:0], experts, 3, fmt, s_x, s_h)
    assert empty["y"].shape == (0, x.shape[1])
    assert empty["offsets"].tolist() == [0, 0, 0, 0] and empty["counts"].tolist() == [0, 0, 0]
    full = moe.forward(x, lg, experts, 3, fmt, s_x, s_h)
    assert full["counts"].tolist() == [5, 5, 5]
    assert full["offsets"].tolist() == [0, 128, 256, 384]
    for e in range(3):
        slots = full["sorted_slots"][128 * e:128 * e + 5]
        assert (slots // 3).tolist() == [0, 1, 2, 3, 4]
    sel = np.take_along_axis(lg.astype(np.float64), full["topk_ids"].astype(np.int64), axis=1)
    ref = np.exp(sel - sel[:, :1])
    np.testing.assert_allclose(full["topk_w"], ref / ref.sum(1, keepdims=True), rtol=4e-7)
    np.testing.assert_allclose(full["topk_w"].sum(1), 1.0, rtol=1e-6)
    one = moe.forward(x[2:3], lg[2:3], experts, 3, fmt, s_x, s_h)
    tok = moe.forward_tokens(x[2:3], lg[2:3], experts, 3, fmt, s_x, s_h)
    np.testing.assert_array_equal(one["y"], tok["y"])      # same sums in the same order



# ---------------------------------------------------------------- BF16 experts with LoRA adapters

def _grid_vals(rng, shape, step, lim):
    n = int(round(lim / step))
    return (rng.integers(-n, n + 1, shape) * step).astype(np.float64)


def test_lora_project_against_exact_rational_sums():
    """a W^T + s (a A^T) B^T against sums of fractions, on grid values."""
    from fractions import Fraction
    rng = np.random.default_rng(21)
    a = _grid_vals(rng, (3, 8), 0.25, 2.0)
    w = _grid_vals(rng, (5, 8), 0.125, 1.0)
    la = _grid_vals(rng, (2, 8), 0.5, 1.0)
    lb = _grid_vals(rng, (5, 2), 0.25, 1.0)
    s = 0.75
    got = moe.lora_project(a, w, la, lb, s)
    for i in range(3):
        for n in range(5):
            main = sum(Fraction(a[i, kk]) * Fraction(w[n, kk]) for kk in range(8))
            z = [sum(Fraction(a[i, kk]) * Fraction(la[j, kk]) for kk in range(8)) for j in range(2)]
            ref = main + Fraction(s) * sum(z[j] * Fraction(lb[n, j]) for j in range(2))
            assert got[i, n] == float(ref), (i, n)


def test_lora_zero_b_is_the_plain_projection():
    rng = np.random.default_rng(22)
    a, w = rng.standard_normal((4, 16)), rng.standard_normal((6, 16))
    la = rng.standard_normal((3, 16))
    np.testing.assert_array_equal(moe.lora_project(a, w, la, np.zeros((6, 3)), 2.0), a @ w.T)
    np.testing.assert_array_equal(moe.lora_project(a, w, None, None, 2.0), a @ w.T)


def test_lora_rank_one_closed_form():
    """A = unit row e_i, B = column c: the update adds s * a[:, i] * c."""
    rng = np.random.default_rng(23)
    a = _grid_vals(rng, (4, 10), 0.25, 2.0)
    w = _grid_vals(rng, (7, 10), 0.25, 1.0)
    c = _grid_vals(rng, (7, 1), 0.5, 2.0)
    la = np.zeros((1, 10))
    la[0, 6] = 1.0
    got = moe.lora_project(a, w, la, c, 0.5)
    np.testing.assert_array_equal(got, a @ w.T + 0.5 * a[:, 6:7] * c[:, 0][None, :])


def test_bf16_layer_with_adapters_equals_merged_weights_written_out():
    """One expert, k = 1: the layer equals a per-token SwiGLU FFN with the
    adapters merged into the weights (W + s B A), written out with math.exp
    and torch's bf16 rounding of the intermediate."""
    import torch
    rng = np.random.default_rng(24)
    T, H, I, r, s = 12, 16, 8, 2, 0.5
    x = _grid_vals(rng, (T, H), 0.25, 2.0).astype(np.float32)
    w = {"gate": _grid_vals(rng, (I, H), 0.125, 0.5), "up": _grid_vals(rng, (I, H), 0.125, 0.5),
         "down": _grid_vals(rng, (H, I), 0.125, 0.5)}
    lo = {m: (_grid_vals(rng, (r, w[m].shape[1]), 0.25, 0.5), _grid_vals(rng, (w[m].shape[0], r), 0.25, 0.5))
          for m in w}
    lg = np.zeros((T, 1), dtype=np.float32)
    res = moe.forward_bf16(x, lg, {0: w}, {0: lo}, 1, s, 1)
    merged = {m: w[m] + s * lo[m][1] @ lo[m][0] for m in w}
    for t in range(T):
        g = [float(np.dot(x[t].astype(np.float64), merged["gate"][i])) for i in range(I)]
        u = [float(np.dot(x[t].astype(np.float64), merged["up"][i])) for i in range(I)]
        h = torch.tensor([gi * ui / (1.0 + math.exp(-gi)) for gi, ui in zip(g, u)], dtype=torch.float64)
        h = h.to(torch.bfloat16).double().numpy()
        o = merged["down"] @ h
        yt = torch.tensor(o, dtype=torch.float64).to(torch.bfloat16).double().numpy()
        np.testing.assert_allclose(res["gate"][t], g, rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(res["y"][t], yt, rtol=2.0 ** -8, atol=1e-30)
        assert np.mean(res["y"][t] == yt) >= 0.9
