"""ctypes binding of libmoe_b200.so (argument marshalling only).

Every function here has the name of the C entry point it calls and takes
PyTorch tensors where the C ABI takes device pointers; it passes their
data_ptr() and the current CUDA stream, and raises MoeError on a non-OK
status.  All arithmetic of the layer runs in the library's CUDA kernels;
there is no fallback: if the shared library is missing, every call raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_NVFP4 = 0
MOE_MXFP8 = 1
MOE_BF16 = 2
FORMATS = {"nvfp4": MOE_NVFP4, "mxfp8": MOE_MXFP8, "bf16": MOE_BF16}

MOE_DEVICE_TIMEOUT_PRODUCER = 0x1
MOE_DEVICE_TIMEOUT_MMA = 0x2
MOE_DEVICE_TIMEOUT_EPILOGUE = 0x4
MOE_DEVICE_TIMEOUT_SELFTEST = 0x8
MOE_DEVICE_BAD_GROUP_EXPERT = 0x10


class MoeError(RuntimeError):
    def __init__(self, name, status, msg):
        super().__init__(f"{name} failed: status {status} ({msg})")
        self.status = status


class moe_config(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("d_ffn", ctypes.c_int32), ("fmt", ctypes.c_int32)]


class moe_weights_layout(ctypes.Structure):
    _fields_ = [("w13_codes", ctypes.c_int64), ("w13_sf", ctypes.c_int64), ("w2_codes", ctypes.c_int64),
                ("w2_sf", ctypes.c_int64), ("scales", ctypes.c_int64), ("total_bytes", ctypes.c_int64)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_CFG = ctypes.POINTER(moe_config)

# name -> (restype, argtypes)
SIGNATURES = {
    "moe_check_config": (ctypes.c_int, [_CFG]),
    "moe_get_weights_layout": (ctypes.c_int, [_CFG, ctypes.POINTER(moe_weights_layout)]),
    "moe_max_rows": (_I64, [_CFG, _I64]),
    "moe_codes_bytes": (_I64, [_CFG, _I64, _I64]),
    "moe_sf_bytes": (_I64, [_CFG, _I64, _I64]),
    "moe_sf_offset": (_I64, [_I64, _I64, _I64]),
    "moe_route_workspace_bytes": (_I64, [_CFG, _I64]),
    "moe_quantize_weights": (ctypes.c_int, [_CFG, _I32, _I32, _P, _P, _P, _P, _P]),
    "moe_route_topk": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P]),
    "moe_router_topk": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _P]),
    "moe_permute": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward_gateup": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward_down": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward_grouped": (ctypes.c_int, [_CFG, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           _P]),
    "moe_pack_weights_bf16": (ctypes.c_int, [_CFG, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32,
                                             ctypes.c_float, _P, _P]),
    "moe_unpermute_combine": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P]),
    "moe_route_topk_noalloc": (ctypes.c_int, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [_P, _I64, _P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def lib():
    """Load libmoe_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m fp8_moe_expert_top_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def make_config(num_experts, top_k, d_model, d_ffn, fmt):
    if isinstance(fmt, str):
        fmt = FORMATS[fmt]
    return moe_config(int(num_experts), int(top_k), int(d_model), int(d_ffn), int(fmt))


def _marshal(name, stream, *tensors):
    """Device pointers of `tensors` (None stays NULL) and the stream handle.

    Every tensor must be a contiguous CUDA tensor on the stream's device, and
    the stream must belong to the current device (the current stream of the
    current device when `stream` is None): the library takes raw device
    pointers and launches on the current device, so a host tensor, a strided
    view, another GPU's memory or another GPU's stream is refused here,
    before anything is enqueued.
    """
    for i, t in enumerate(tensors):
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: argument {i} is on {t.device}, a CUDA tensor is required")
        if not t.is_contiguous():
            raise ValueError(f"{name}: argument {i} is not contiguous")
    s = torch.cuda.current_stream() if stream is None else stream
    if s.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: the stream is on {s.device} but the current device is "
                         f"cuda:{torch.cuda.current_device()} (the library launches on the current device)")
    for i, t in enumerate(tensors):
        if t is not None and t.device != s.device:
            raise ValueError(f"{name}: argument {i} is on {t.device}, the stream on {s.device}")
    return [None if t is None else ctypes.c_void_p(t.data_ptr()) for t in tensors], ctypes.c_void_p(s.cuda_stream)


def _check(name, status):
    if status != 0:
        raise MoeError(name, status, lib().moe_status_string(status).decode())


# ----------------------------------------------------------------- sizes

def moe_check_config(cfg):
    return lib().moe_check_config(ctypes.byref(cfg))


def moe_get_weights_layout(cfg):
    out = moe_weights_layout()
    _check("moe_get_weights_layout", lib().moe_get_weights_layout(ctypes.byref(cfg), ctypes.byref(out)))
    return out


def moe_max_rows(cfg, T):
    return lib().moe_max_rows(ctypes.byref(cfg), int(T))


def moe_codes_bytes(cfg, rows, K):
    return lib().moe_codes_bytes(ctypes.byref(cfg), int(rows), int(K))


def moe_sf_bytes(cfg, rows, K):
    return lib().moe_sf_bytes(ctypes.byref(cfg), int(rows), int(K))


def moe_sf_offset(row, col, nsf):
    return lib().moe_sf_offset(int(row), int(col), int(nsf))


def moe_route_workspace_bytes(cfg, T):
    return lib().moe_route_workspace_bytes(ctypes.byref(cfg), int(T))


# ----------------------------------------------------------------- calls

def moe_quantize_weights(cfg, expert_begin, expert_count, w_gate, w_up, w_down, packed, stream=None):
    (wg, wu, wd, pk), st = _marshal("moe_quantize_weights", stream, w_gate, w_up, w_down, packed)
    _check("moe_quantize_weights", lib().moe_quantize_weights(
        ctypes.byref(cfg), int(expert_begin), int(expert_count), wg, wu, wd, pk, st))


def moe_route_topk(cfg, T, logits, topk_ids, topk_w, expert_counts, expert_offsets, sorted_slots, slot_to_row,
                   workspace, stream=None):
    p, st = _marshal("moe_route_topk", stream, logits, topk_ids, topk_w, expert_counts, expert_offsets,
                     sorted_slots, slot_to_row, workspace)
    _check("moe_route_topk", lib().moe_route_topk(
        ctypes.byref(cfg), int(T), *p, int(workspace.numel() * workspace.element_size()), st))


def moe_route_topk_noalloc(cfg, T, logits, topk_ids, topk_w, expert_counts, expert_offsets, sorted_slots,
                           slot_to_row, stream=None):
    """moe_route_topk without a workspace, for callers that cannot allocate
    device memory (the library's fixed 4 MiB scratch array is used instead)."""
    p, st = _marshal("moe_route_topk_noalloc", stream, logits, topk_ids, topk_w, expert_counts, expert_offsets,
                     sorted_slots, slot_to_row)
    _check("moe_route_topk_noalloc", lib().moe_route_topk_noalloc(ctypes.byref(cfg), int(T), *p, st))


def moe_router_topk(cfg, T, x, w_router, logits_out, topk_ids, topk_w, expert_counts, expert_offsets, sorted_slots,
                    slot_to_row, workspace, status_word=None, stream=None):
    """Routing from bf16 x [T, H] and bf16 router weights [E, H]; logits_out
    (float32 [T, E]) is an optional copy of the scores."""
    p, st = _marshal("moe_router_topk", stream, x, w_router, logits_out, topk_ids, topk_w, expert_counts,
                     expert_offsets, sorted_slots, slot_to_row, workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    status = _marshal("moe_router_topk", stream, status_word)[0][0]
    _check("moe_router_topk", lib().moe_router_topk(ctypes.byref(cfg), int(T), *p, ws_bytes, status, st))


def moe_permute(cfg, T, x, act_scale, slot_to_row, a_codes, a_sf, stream=None):
    p, st = _marshal("moe_permute", stream, x, act_scale, slot_to_row, a_codes, a_sf)
    _check("moe_permute", lib().moe_permute(ctypes.byref(cfg), int(T), *p, st))


def moe_forward(cfg, T, packed, a_codes, a_sf, act_scale, inter_scale, expert_offsets, expert_counts, h_codes, h_sf,
                down_out, gateup_debug=None, status_word=None, stream=None):
    p, st = _marshal("moe_forward", stream, packed, a_codes, a_sf, act_scale, inter_scale, expert_offsets,
                     expert_counts, h_codes, h_sf, down_out, gateup_debug, status_word)
    _check("moe_forward", lib().moe_forward(ctypes.byref(cfg), int(T), *p, st))


def moe_forward_gateup(cfg, T, packed, a_codes, a_sf, act_scale, inter_scale, expert_offsets, expert_counts,
                       h_codes, h_sf, gateup_debug=None, status_word=None, stream=None):
    p, st = _marshal("moe_forward_gateup", stream, packed, a_codes, a_sf, act_scale, inter_scale, expert_offsets,
                     expert_counts, h_codes, h_sf, gateup_debug, status_word)
    _check("moe_forward_gateup", lib().moe_forward_gateup(ctypes.byref(cfg), int(T), *p, st))


def moe_forward_down(cfg, T, packed, h_codes, h_sf, inter_scale, expert_offsets, expert_counts, down_out,
                     status_word=None, stream=None):
    p, st = _marshal("moe_forward_down", stream, packed, h_codes, h_sf, inter_scale, expert_offsets, expert_counts,
                     down_out, status_word)
    _check("moe_forward_down", lib().moe_forward_down(ctypes.byref(cfg), int(T), *p, st))


def moe_forward_grouped(cfg, num_groups, max_rows, packed, a_codes, a_sf, act_scale, inter_scale, group_offsets,
                        group_counts, group_expert, h_codes, h_sf, down_out, gateup_debug=None, status_word=None,
                        stream=None):
    p, st = _marshal("moe_forward_grouped", stream, packed, a_codes, a_sf, act_scale, inter_scale, group_offsets,
                     group_counts, group_expert, h_codes, h_sf, down_out, gateup_debug, status_word)
    _check("moe_forward_grouped", lib().moe_forward_grouped(ctypes.byref(cfg), int(num_groups), int(max_rows), *p,
                                                            st))


def moe_pack_weights_bf16(cfg, expert_begin, expert_count, w_gate, w_up, w_down, lora=None, lora_rank=0,
                          lora_scaling=0.0, packed=None, stream=None):
    """bf16 weights [n, I, H] / [n, H, I] and optional adapters
    lora = (a_gate, b_gate, a_up, b_up, a_down, b_down) into packed."""
    lo = lora if lora is not None else (None,) * 6
    p, st = _marshal("moe_pack_weights_bf16", stream, w_gate, w_up, w_down, *lo, packed)
    _check("moe_pack_weights_bf16", lib().moe_pack_weights_bf16(
        ctypes.byref(cfg), int(expert_begin), int(expert_count), *p[:9], int(lora_rank), float(lora_scaling), p[9],
        st))


def moe_unpermute_combine(cfg, T, down_out, topk_w, slot_to_row, y, stream=None):
    p, st = _marshal("moe_unpermute_combine", stream, down_out, topk_w, slot_to_row, y)
    _check("moe_unpermute_combine", lib().moe_unpermute_combine(ctypes.byref(cfg), int(T), *p, st))


def moe_selftest_bounded_wait(status_word, limit_ns, stream=None):
    (sw,), st = _marshal("moe_selftest_bounded_wait", stream, status_word)
    _check("moe_selftest_bounded_wait", lib().moe_selftest_bounded_wait(sw, int(limit_ns), st))
