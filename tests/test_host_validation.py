"""Host-side argument checks of the binding and the layer (CPU only).

The library takes raw device pointers, so the binding refuses host tensors
before anything reaches it, and the layer refuses a non-CUDA device.  These
checks run before any CUDA call, so they hold on a machine without a GPU.
"""

import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from fp8_moe_expert_top_b200.layer import ExpertLayer

CFG = B.make_config(8, 2, 256, 128, "nvfp4")


def _host(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


CALLS = {
    "moe_quantize_weights": lambda h: B.moe_quantize_weights(CFG, 0, 1, h, h, h, h),
    "moe_route_topk": lambda h: B.moe_route_topk(CFG, 4, h, h, h, h, h, h, h, h),
    "moe_route_topk_noalloc": lambda h: B.moe_route_topk_noalloc(CFG, 4, h, h, h, h, h, h, h),
    "moe_router_topk": lambda h: B.moe_router_topk(CFG, 4, h, h, h, h, h, h, h, h, h, h, h),
    "moe_permute": lambda h: B.moe_permute(CFG, 4, h, h, h, h, h),
    "moe_forward": lambda h: B.moe_forward(CFG, 4, h, h, h, h, h, h, h, h, h, h),
    "moe_forward_gateup": lambda h: B.moe_forward_gateup(CFG, 4, h, h, h, h, h, h, h, h, h),
    "moe_forward_down": lambda h: B.moe_forward_down(CFG, 4, h, h, h, h, h, h, h),
    "moe_forward_grouped": lambda h: B.moe_forward_grouped(CFG, 2, 128, h, h, h, h, h, h, h, h, h, h, h),
    "moe_pack_weights_bf16": lambda h: B.moe_pack_weights_bf16(CFG, 0, 1, h, h, h, packed=h),
    "moe_unpermute_combine": lambda h: B.moe_unpermute_combine(CFG, 4, h, h, h, h),
    "moe_selftest_bounded_wait": lambda h: B.moe_selftest_bounded_wait(h, 1000),
}


def test_every_compute_call_is_covered():
    sizes = {"moe_check_config", "moe_get_weights_layout", "moe_max_rows", "moe_codes_bytes", "moe_sf_bytes",
             "moe_sf_offset", "moe_route_workspace_bytes", "moe_status_string"}
    assert set(CALLS) == set(B.SIGNATURES) - sizes


@pytest.mark.parametrize("name", sorted(CALLS))
def test_binding_refuses_host_tensors(name):
    with pytest.raises(ValueError, match="a CUDA tensor is required"):
        CALLS[name](_host(64))


def test_layer_refuses_a_host_device():
    with pytest.raises(ValueError, match="CUDA device"):
        ExpertLayer(8, 2, 256, 128, "nvfp4", 16, "cpu", s_x=1.0, s_h=1.0)


def _unbuilt_layer(T_max=64, H=256, E=8):
    """An ExpertLayer shell with the attributes the host checks read (no
    device buffers), for exercising those checks without a GPU."""
    layer = object.__new__(ExpertLayer)
    layer.H, layer.E, layer.T_max = H, E, T_max
    layer.device = torch.device("cuda", 0)
    return layer


def test_layer_forward_checks_run_before_any_launch():
    layer = _unbuilt_layer()
    T, H, E = 64, 256, 8
    x = _host(T, H, dtype=torch.bfloat16)
    lg = _host(T, E)
    with pytest.raises(ValueError, match="buffers hold"):
        layer.forward(_host(T + 1, H, dtype=torch.bfloat16), _host(T + 1, E))
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, lg.double())
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, _host(T, E - 1))
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, lg[:T - 1])
    with pytest.raises(ValueError, match="^x: "):
        layer.forward(x.float(), lg)
    with pytest.raises(ValueError, match="^x: "):
        layer.forward(_host(T, H, 1, dtype=torch.bfloat16), lg)
    with pytest.raises(ValueError, match="is on cpu"):
        layer.forward(x, lg)


def test_forward_graph_uses_the_graphs_own_token_count():
    import types
    layer, other = _unbuilt_layer(), _unbuilt_layer()
    x, lg = _host(64, 256, dtype=torch.bfloat16), _host(64, 8)
    g = types.SimpleNamespace(moe_layer_io=(layer, 37, None, None, None))
    with pytest.raises(ValueError, match="captured for T = 37"):
        layer.forward_graph(g, x, lg)
    with pytest.raises(ValueError, match="not captured by this layer"):
        other.forward_graph(g, x, lg)
    with pytest.raises(ValueError, match="not captured by this layer"):
        layer.forward_graph(types.SimpleNamespace(), x, lg)


def test_capture_stack_refuses_an_empty_stack():
    from fp8_moe_expert_top_b200.layer import capture_stack
    with pytest.raises(ValueError, match="at least one pass"):
        capture_stack([], _host(4, 256, dtype=torch.bfloat16), [None, None], 4)


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers: run only where nothing can launch")
@pytest.mark.parametrize("T", [-1, (1 << 20) + 1])
def test_token_count_out_of_range_is_refused_before_any_launch(T):
    """T outside 0..2^20 returns MOE_ERR_UNSUPPORTED from every call that takes
    T; the pointers (placeholders, never dereferenced) are not looked at."""
    import ctypes
    L = B.lib()
    cfg = ctypes.byref(CFG)
    p = ctypes.c_void_p(0x10000)
    calls = {
        "moe_route_topk": lambda: L.moe_route_topk(cfg, T, p, p, p, p, p, p, p, p, 1 << 30, None),
        "moe_route_topk_noalloc": lambda: L.moe_route_topk_noalloc(cfg, T, p, p, p, p, p, p, p, None),
        "moe_router_topk": lambda: L.moe_router_topk(cfg, T, p, p, None, p, p, p, p, p, p, p, 1 << 30, None, None),
        "moe_permute": lambda: L.moe_permute(cfg, T, p, p, p, p, p, None),
        "moe_forward": lambda: L.moe_forward(cfg, T, p, p, p, p, p, p, p, p, p, p, None, None, None),
        "moe_forward_gateup": lambda: L.moe_forward_gateup(cfg, T, p, p, p, p, p, p, p, p, p, None, None, None),
        "moe_forward_down": lambda: L.moe_forward_down(cfg, T, p, p, p, p, p, p, p, None, None),
        "moe_unpermute_combine": lambda: L.moe_unpermute_combine(cfg, T, p, p, p, p, None),
    }
    for name, call in calls.items():
        assert call() == 2, name                      # MOE_ERR_UNSUPPORTED
    assert B.moe_max_rows(CFG, T) == -1
    assert B.moe_route_workspace_bytes(CFG, T) == -1
