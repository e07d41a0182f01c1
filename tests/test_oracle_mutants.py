"""Planted mistakes in the oracle must each fail one of its pins (CPU only).

Each case below rebuilds one oracle function from its source with a single
plausible mistake (a dropped term, a wrong sign, bias or index, a tie broken
the other way, a transposed operand, a missing rounding), installs it in
place of the original and runs the pins of test_oracle_formats.py and
test_oracle_route_moe.py.  The case passes when at least one pin fails, which
shows that the pins would notice that mistake in the oracle.  The mutants
live only here, on the CPU; the oracle itself is never edited.

Every edit names a fragment that must occur exactly once in the function's
current source, so a change to the oracle that removes the fragment fails
loudly here instead of silently testing nothing.
"""

import functools
import inspect
import textwrap

import pytest

import test_oracle_formats as pins_formats
import test_oracle_route_moe as pins_route_moe
from oracle import formats as fm
from oracle import moe
from oracle import route as rt

# Pins that take a second or more each run last.
_SLOW = ("test_nvfp4_choice_against_exact_rational_search", "test_nvfp4_against_brute_force_over_all_scales")


def _pins():
    """Every pin function of the two pin modules, parametrizations expanded."""
    out = []
    for mod in (pins_formats, pins_route_moe):
        for name, fn in vars(mod).items():
            if not name.startswith("test_") or not callable(fn) or getattr(fn, "__module__", None) != mod.__name__:
                continue
            marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
            if not marks:
                out.append((name, fn))
                continue
            assert len(marks) == 1, name
            argname, values = marks[0].args
            for v in values:
                out.append((f"{name}[{v}]", functools.partial(fn, **{argname: v})))
    out.sort(key=lambda p: p[0].split("[")[0] in _SLOW)
    return out


PINS = _pins()


def _rebuild(module, name, old, new):
    """`module.name` recompiled from its source with `old` replaced by `new`."""
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    assert src.count(old) == 1, f"{module.__name__}.{name}: fragment {old!r} occurs {src.count(old)} times"
    ns = dict(vars(module))
    exec(compile(src.replace(old, new), f"<mutant of {module.__name__}.{name}>", "exec"), ns)
    return ns[name]


# (id, module, function, fragment, replacement)
MUTANTS = [
    # E2M1
    ("e2m1_decode_sign_flipped", fm, "e2m1_decode", "-mag, mag", "mag, -mag"),
    ("e2m1_decode_wrong_magnitude_index", fm, "e2m1_decode", "[codes & 7]", "[(codes >> 1) & 7]"),
    ("e2m1_tie_2p5_rounds_up", fm, "e2m1_encode_magnitude", "v > 2.5, 5", "v >= 2.5, 5"),
    ("e2m1_tie_0p25_rounds_up", fm, "e2m1_encode_magnitude", "v > 0.25, 1", "v >= 0.25, 1"),
    ("e2m1_tie_5_rounds_up", fm, "e2m1_encode_magnitude", "v > 5.0, 7", "v >= 5.0, 7"),
    # E4M3
    ("e4m3_decode_bias_8", fm, "e4m3_decode", "exp.astype(np.float64) - 7.0", "exp.astype(np.float64) - 8.0"),
    ("e4m3_decode_subnormal_step", fm, "e4m3_decode", "(man / 8.0) * 2.0 ** -6", "(man / 8.0) * 2.0 ** -7"),
    ("e4m3_decode_no_nan", fm, "e4m3_decode", "(codes & 0x7F) == 0x7F", "(codes & 0x7F) == 0x80"),
    ("e4m3_encode_ties_away", fm, "e4m3_encode", "np.rint(frac8)", "np.floor(frac8 + 0.5)"),
    ("e4m3_encode_subnormal_ties_away", fm, "e4m3_encode", "np.rint(a * 2.0 ** 9)", "np.floor(a * 2.0 ** 9 + 0.5)"),
    ("e4m3_encode_saturates_to_nan", fm, "e4m3_encode", "a >= E4M3_MAX, 0x7E", "a >= E4M3_MAX, 0x7F"),
    ("e4m3_encode_negative_zero", fm, "e4m3_encode", "np.where(mag == 0, 0, mag | (sign << 7))",
     "mag | (sign << 7)"),
    ("e4m3_encode_truncates", fm, "e4m3_encode", "np.rint(frac8)", "np.floor(frac8)"),
    # E8M0
    ("e8m0_decode_bias_128", fm, "e8m0_decode", "- 127.0", "- 128.0"),
    # float32 helpers
    ("error_sum_left_to_right", fm, "pairwise_tree_sum_f32",
     "while s.shape[-1] > 1:\n        s = (s[..., 0::2] + s[..., 1::2]).astype(np.float32)\n    return s[..., 0]",
     "return np.cumsum(s, axis=-1, dtype=np.float32)[..., -1]"),
    # NVFP4
    ("tensor_scale_divisor_448", fm, "nvfp4_tensor_scale", "F32(NVFP4_TENSOR_DIVISOR)", "F32(448.0)"),
    ("tensor_scale_zero_not_one", fm, "nvfp4_tensor_scale", "return F32(1.0)", "return F32(0.0)"),
    ("candidate_drops_tensor_scale_in_code", fm, "_nvfp4_candidate", "denom = (F32(c) * s_g)",
     "denom = (F32(c) * F32(1.0))"),
    ("candidate_drops_tensor_scale_in_effective_scale", fm, "_nvfp4_candidate",
     "S_c = (_f32(e4m3_decode(e_c)) * s_g)", "S_c = (_f32(e4m3_decode(e_c)) * F32(1.0))"),
    ("candidate_absolute_error", fm, "_nvfp4_candidate", "pairwise_tree_sum_f32((d * d)",
     "pairwise_tree_sum_f32((np.abs(d))"),
    ("candidate_error_in_scaled_domain", fm, "_nvfp4_candidate", "d = (x - recon)", "d = (x - recon) / S_safe"),
    ("candidate_negative_zero_code", fm, "_nvfp4_candidate", "neg = (x < 0) & (mag != 0)", "neg = (x < 0)"),
    ("candidate_codes_unscaled", fm, "_nvfp4_candidate", "(np.abs(x) / S_safe)", "(np.abs(x) * S_safe)"),
    ("four_wins_ties", fm, "nvfp4_quantize_blocks", "four = err4 < err6", "four = err4 <= err6"),
    ("keeps_the_worse_candidate", fm, "nvfp4_quantize_blocks", "four = err4 < err6", "four = err4 > err6"),
    ("block_max_signed", fm, "nvfp4_quantize_blocks", "np.max(np.abs(x), axis=-1)", "np.max(x, axis=-1)"),
    ("only_six_candidate", fm, "nvfp4_quantize_blocks", "four = err4 < err6", "four = err4 < -1.0"),
    ("dequant_drops_tensor_scale", fm, "nvfp4_dequantize_rows", "* float(F32(s_g))", "* 1.0"),
    # MXFP8
    ("mx_scale_emax_7", fm, "mxfp8_scale_exponent", "fl - E4M3_EMAX + 127", "fl - 7 + 127"),
    ("mx_scale_ceil_log2", fm, "mxfp8_scale_exponent", "fl = e2 - 1", "fl = e2"),
    ("mx_scale_no_clamp_low", fm, "mxfp8_scale_exponent", "np.clip(fl - E4M3_EMAX + 127, 0, 254)",
     "np.clip(fl - E4M3_EMAX + 127, 1, 254)"),
    ("mx_quant_scale_inverted", fm, "mxfp8_quantize_blocks", "np.exp2(127.0 - e", "np.exp2(-127.0 + e"),
    ("mx_dequant_divides", fm, "mxfp8_dequantize_rows", "v * e8m0_decode(scales)", "v / e8m0_decode(scales)"),
    # bfloat16 rounding
    ("bf16_truncates", fm, "bf16_round", "np.rint(a / ulp)", "np.floor(a / ulp)"),
    ("bf16_nine_bits", fm, "bf16_round", "E.astype(np.float64) - 7.0", "E.astype(np.float64) - 8.0"),
    ("bf16_ties_away", fm, "bf16_round", "np.rint(a / ulp)", "np.floor(a / ulp + 0.5)"),
    # exp and routing
    ("exp_drops_low_ln2", rt, "exp_own", "(n * LN2_LO_F32)", "(n * F32(0.0))"),
    ("exp_short_polynomial", rt, "exp_own", "range(6, -1, -1)", "range(5, -1, -1)"),
    ("exp_no_underflow_cut", rt, "exp_own", "x < EXP_UNDERFLOW_F32", "x < F32(-1000.0)"),
    ("topk_ties_to_higher_index", rt, "topk_select", "best = np.argmax(work, axis=1)",
     "best = work.shape[1] - 1 - np.argmax(work[:, ::-1], axis=1)"),
    ("topk_smallest", rt, "topk_select", "best = np.argmax(work, axis=1)", "best = np.argmin(work, axis=1)"),
    ("softmax_unnormalised", rt, "topk_softmax", "return (e / s[:, None])", "return (e / 1.0)"),
    ("softmax_drops_last_term", rt, "topk_softmax", "for j in range(1, k):", "for j in range(1, k - 1):"),
    ("softmax_of_all_logits_max", rt, "topk_softmax", "m = sel[:, :1]", "m = sel[:, :1] * 0.0"),
    ("slots_unpadded", rt, "sort_slots", "round_up(counts[e], ROW_ALIGN)", "counts[e]"),
    ("slots_descending_tokens", rt, "sort_slots", "for s in range(T * k):", "for s in reversed(range(T * k)):"),
    ("slots_inverse_off_by_one", rt, "sort_slots", "slot_to_row[s] = row", "slot_to_row[s] = row + 1"),
    # permute, FFN, combine
    ("permute_token_index_mod", moe, "permute_quantize", "sorted_slots // k", "sorted_slots % k"),
    ("swiglu_wrong_sign", moe, "swiglu", "np.exp(-g)", "np.exp(g)"),
    ("swiglu_gates_on_up", moe, "swiglu", "np.exp(-g)", "np.exp(-u)"),
    ("ffn_gate_reads_up", moe, "expert_ffn", "g = a_deq @ wq_deq[\"gate\"].T", "g = a_deq @ wq_deq[\"up\"].T"),
    ("ffn_swiglu_operands_swapped", moe, "expert_ffn", "swiglu(g, u)", "swiglu(u, g)"),
    ("ffn_skips_h_requantization", moe, "expert_ffn", "out = h_deq @", "out = h.astype(np.float64) @"),
    ("ffn_h_not_rounded_to_f32", moe, "expert_ffn", "h = swiglu(g, u).astype(np.float32)",
     "h = swiglu(g, u).astype(np.float16).astype(np.float32)"),
    ("combine_unweighted", moe, "combine", "y += topk_w[:, j].astype(np.float64)[:, None] * out_rows[rows]",
     "y += out_rows[rows]"),
    ("combine_transposed_slots", moe, "combine", "slot_to_row.reshape(T, k)[:, j]", "slot_to_row.reshape(k, T)[j, :]"),
    ("combine_no_bf16_rounding", moe, "combine", "return fm.bf16_round(y)", "return y"),
    ("forward_activation_scale_s_h", moe, "forward", "a_sf[lo:lo + cnt], fmt, s_x)", "a_sf[lo:lo + cnt], fmt, s_h)"),
    ("forward_intermediate_scale_s_x", moe, "forward", "expert_ffn(a_deq, wq, fmt, s_h)",
     "expert_ffn(a_deq, wq, fmt, s_x)"),
    ("weight_tensor_scale_signed_max", moe, "weight_tensor_scale", "np.max(np.abs(np.asarray(w, dtype=np.float32)))",
     "np.max(np.asarray(w, dtype=np.float32))"),
    # router scores
    ("router_logits_float32_sum", rt, "router_logits", "(x64 @ w64.T)",
     "(x64.astype(np.float32) @ w64.astype(np.float32).T)"),
    ("router_logits_experts_reversed", rt, "router_logits", "w64 = np.asarray(w_router, dtype=np.float64)",
     "w64 = np.asarray(w_router, dtype=np.float64)[::-1]"),
    ("router_logits_no_float32_rounding", rt, "router_logits", ".astype(np.float32)", ""),
    # BF16 experts with adapters
    ("lora_scaling_dropped", moe, "lora_project", "float(scaling) * ", ""),
    ("lora_b_not_transposed", moe, "lora_project", "np.asarray(lora_b, dtype=np.float64).T",
     "np.asarray(lora_b, dtype=np.float64)"),
    ("lora_down_input_not_bf16", moe, "expert_ffn_bf16", "h = fm.bf16_round(swiglu(g, u))", "h = swiglu(g, u)"),
    ("lora_up_uses_gate_adapter", moe, "expert_ffn_bf16", 'lo.get("up", (None, None))', 'lo.get("gate", (None, None))'),
]


def test_mutant_ids_unique():
    ids = [m[0] for m in MUTANTS]
    assert len(ids) == len(set(ids))


def test_pins_pass_unmutated():
    """The harness itself: every pin passes on the oracle as it stands."""
    for name, pin in PINS:
        pin()


@pytest.mark.filterwarnings("ignore::RuntimeWarning")     # overflow inside some mutants
@pytest.mark.parametrize("mid,module,func,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, mid, module, func, old, new):
    monkeypatch.setattr(module, func, _rebuild(module, func, old, new))
    for name, pin in PINS:
        try:
            pin()
        except Exception:          # an assertion, or the mutant breaking a shape or a check
            return
    pytest.fail(f"no pin fails with the planted mistake {mid} in {module.__name__}.{func}")
