"""GPU parity on small layers, every step against the oracle (GPU).

Workload "tiny": T = 64 tokens, d_model 256, expert ffn 128, 8 experts,
top-2, bf16 x ~ N(0, 1), float32 logits ~ N(0, 1), weights N(0, 1/fan_in)
quantized by the library (NVFP4 with the 4-vs-6 pick, or MXFP8).  Bars:
weight codes, routing, permutation and activation codes bit-exact; gate/up
float32 relative Frobenius error <= 1e-4; at most 1e-3 of the requantized
intermediate (code, block scale) pairs differ; bf16 output relative
Frobenius error <= 1e-2.  Edge cases: a single token, routing that leaves
experts empty or sends every token to the same experts, tied logits.
"""

import dataclasses

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from fp8_moe_expert_top_b200 import inputs
from oracle import moe as omoe

from gpu_common import assert_expert_equal, build_layer, gpu_expert, oracle_expert
from helpers import ACT_TR, rel_fro, sfvec, tiled_codes, unswizzle_sf

TINY = inputs.WORKLOADS["tiny_nvfp4"]
TINY_MX = dataclasses.replace(TINY, name="tiny_mxfp8", fmt=inputs.MXFP8)
# T * k > 128 * E: the prefill shape class (several 128-row blocks per expert)
TINY_PREFILL = dataclasses.replace(TINY, name="tiny_nvfp4_prefill", T=1024)
TINY_PREFILL_MX = dataclasses.replace(TINY_PREFILL, name="tiny_mxfp8_prefill", fmt=inputs.MXFP8)

_layers = {}


def get_layer(wl, dev):
    key = (wl.name, wl.T)
    if key not in _layers:
        _layers[key] = build_layer(wl, dev)
    return _layers[key]


def oracle_experts(wl):
    return {e: oracle_expert(wl, e, "cpu") for e in range(wl.num_experts)}


def run_and_compare(layer, wl, x, logits, experts_q):
    dev = layer.device
    T = x.shape[0]
    layer.status.zero_()
    layer.gateup_debug.fill_(float("nan"))
    y = layer.forward(x.to(dev), logits.to(dev))
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = omoe.forward(x.float().numpy(), logits.numpy(), experts_q, wl.top_k, wl.fmt,
                       inputs.S_X, inputs.S_H, wl.num_experts)
    # routing: bit-exact
    np.testing.assert_array_equal(layer.topk_ids[:T].cpu().numpy(), ref["topk_ids"])
    np.testing.assert_array_equal(layer.topk_w[:T].cpu().numpy().view(np.uint32), ref["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(layer.expert_counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(layer.expert_offsets.cpu().numpy(), ref["offsets"])
    R = int(ref["offsets"][-1])
    ss = layer.sorted_slots.cpu().numpy()
    np.testing.assert_array_equal(ss[:R], ref["sorted_slots"])
    R_call = B.moe_max_rows(layer.cfg, T)          # rows this call owns
    assert np.all(ss[R:R_call] == -1)
    np.testing.assert_array_equal(layer.slot_to_row[:T * wl.top_k].cpu().numpy(), ref["slot_to_row"])
    valid = ref["valid"]
    H, I, v = wl.d_model, wl.d_ffn, sfvec(wl.fmt)
    Rb = layer.R_max
    # activation codes: bit-exact on valid rows
    a_codes = tiled_codes(wl.fmt, layer.a_codes.cpu().numpy(), np.arange(R), H, ACT_TR)
    a_sf = unswizzle_sf(layer.a_sf.cpu().numpy(), Rb, H // v)[:R]
    np.testing.assert_array_equal(a_codes[valid], ref["a_codes"][valid])
    np.testing.assert_array_equal(a_sf[valid], ref["a_sf"][valid])
    # gate/up float32
    dbg = layer.gateup_debug.cpu().numpy()[:R]
    err_g = rel_fro(dbg[valid, :I], ref["gate"][valid])
    err_u = rel_fro(dbg[valid, I:], ref["up"][valid])
    assert err_g <= 1e-4 and err_u <= 1e-4, (err_g, err_u)
    assert np.all(np.isnan(dbg[~valid]))
    # requantized intermediate
    hc = tiled_codes(wl.fmt, layer.h_codes.cpu().numpy(), np.arange(R), I, ACT_TR)
    hs = unswizzle_sf(layer.h_sf.cpu().numpy(), Rb, I // v)[:R]
    rc, rs = ref["h_codes"], ref["h_sf"]
    differ = (hc != rc) | (np.repeat(hs, v, axis=1) != np.repeat(rs, v, axis=1))
    frac = float(differ[valid].mean())
    assert frac <= 1e-3, frac
    # layer output
    yr = ref["y"]
    err_y = rel_fro(y.float().cpu().numpy(), yr)
    assert err_y <= 1e-2, err_y
    return dict(err_g=err_g, err_u=err_u, h_frac=frac, err_y=err_y)


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX], ids=lambda w: w.name)
def test_weights_bit_exact(cuda_device, wl):
    layer = get_layer(wl, cuda_device)
    for e in range(wl.num_experts):
        assert_expert_equal(gpu_expert(layer, wl, e), oracle_expert(wl, e, "cpu"), e)


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX, TINY_PREFILL, TINY_PREFILL_MX], ids=lambda w: w.name)
def test_layer_seeded_inputs(cuda_device, wl):
    layer = get_layer(wl, cuda_device)
    x, lg = inputs.make_x(wl), inputs.make_logits(wl)
    run_and_compare(layer, wl, x, lg, oracle_experts(wl))


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX], ids=lambda w: w.name)
@pytest.mark.parametrize("case", ["one_token", "hot_experts", "ties", "empty_experts", "ragged", "large_logits"])
def test_layer_edge_cases(cuda_device, wl, case):
    layer = get_layer(wl, cuda_device)
    E = wl.num_experts
    if case == "one_token":
        x, lg = inputs.make_x(wl, T=1, seed=11), inputs.make_logits(wl, T=1, seed=12)
    elif case == "hot_experts":          # every token picks experts 3 and 5
        x, lg = inputs.make_x(wl, seed=13), inputs.make_logits(wl, seed=14)
        lg[:, 3] += 50.0
        lg[:, 5] += 40.0
    elif case == "ties":                 # many equal logits, ties go to the lower index
        x = inputs.make_x(wl, seed=15)
        lg = inputs.make_logits_with_ties(wl.T, E, seed=16)
    elif case == "empty_experts":        # experts 0, 1 and 6 never chosen
        x, lg = inputs.make_x(wl, seed=17), inputs.make_logits(wl, seed=18)
        lg[:, [0, 1, 6]] -= 100.0
    elif case == "large_logits":         # rows offset far from zero: exp of a raw logit would overflow
        x, lg = inputs.make_x(wl, seed=21), inputs.make_logits(wl, seed=22)
        offs = torch.tensor([-300.0, 150.0, 1000.0])[torch.arange(wl.T) % 3]
        lg = (lg * 3.0 + offs[:, None]).to(torch.float32)
    else:                                # T not a multiple of anything
        x, lg = inputs.make_x(wl, T=37, seed=19), inputs.make_logits(wl, T=37, seed=20)
    run_and_compare(layer, wl, x, lg, oracle_experts(wl))


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY_PREFILL, TINY_PREFILL_MX], ids=lambda w: w.name)
@pytest.mark.parametrize("case", ["hot_experts", "empty_experts", "ragged", "small_route_limit", "large_route_min"])
def test_prefill_layer_edge_cases(cuda_device, wl, case):
    """Prefill-shaped layer with skewed routing, empty experts and a ragged batch;
    512 tokens is the largest batch routed by the one-CTA small-batch path, 513
    the smallest routed by the bitmap scan / scatter kernels."""
    layer = get_layer(wl, cuda_device)
    if case in ("small_route_limit", "large_route_min"):
        T = 512 if case == "small_route_limit" else 513
        x, lg = inputs.make_x(wl, T=T, seed=29), inputs.make_logits(wl, T=T, seed=30)
    elif case == "hot_experts":
        x, lg = inputs.make_x(wl, seed=23), inputs.make_logits(wl, seed=24)
        lg[:, 3] += 50.0
    elif case == "empty_experts":
        x, lg = inputs.make_x(wl, seed=25), inputs.make_logits(wl, seed=26)
        lg[:, [0, 6]] -= 100.0
    else:
        x, lg = inputs.make_x(wl, T=777, seed=27), inputs.make_logits(wl, T=777, seed=28)
    run_and_compare(layer, wl, x, lg, oracle_experts(wl))


@pytest.mark.gpu
def test_empty_batch(cuda_device):
    layer = get_layer(TINY, cuda_device)
    x = torch.zeros(0, TINY.d_model, dtype=torch.bfloat16, device=cuda_device)
    lg = torch.zeros(0, TINY.num_experts, dtype=torch.float32, device=cuda_device)
    y = layer.forward(x, lg)
    torch.cuda.synchronize()
    assert y.shape == (0, TINY.d_model)
    assert int(layer.expert_offsets[-1].item()) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX], ids=lambda w: w.name)
def test_cuda_graph_replay_matches_eager(cuda_device, wl):
    """The layer captured as one CUDA graph gives the eager results bit for bit."""
    layer = get_layer(wl, cuda_device)
    x, lg = inputs.make_x(wl, seed=31).to(cuda_device), inputs.make_logits(wl, seed=32).to(cuda_device)
    y_eager = layer.forward(x, lg).clone()
    h_eager = layer.h_codes.clone()
    torch.cuda.synchronize()
    g = layer.capture(wl.T)
    for _ in range(2):
        layer.y.zero_()
        y_graph = layer.forward_graph(g, x, lg)
        torch.cuda.synchronize()
        assert torch.equal(y_graph.view(torch.int16), y_eager.view(torch.int16))
    assert torch.equal(layer.h_codes, h_eager)


@pytest.mark.gpu
def test_graphs_of_two_batch_sizes_replay_independently(cuda_device):
    """Each graph remembers its own token count and buffers: a graph captured
    earlier still replays correctly after another one has been captured."""
    wl = TINY
    layer = get_layer(wl, cuda_device)
    x, lg = inputs.make_x(wl, seed=33).to(cuda_device), inputs.make_logits(wl, seed=34).to(cuda_device)
    y_full = layer.forward(x, lg).clone()
    y_part = layer.forward(x[:37], lg[:37]).clone()
    g_full = layer.capture(wl.T)
    g_part = layer.capture(37)
    for _ in range(2):
        y = layer.forward_graph(g_full, x, lg).clone()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_full.view(torch.int16))
        y = layer.forward_graph(g_part, x[:37], lg[:37]).clone()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_part.view(torch.int16))
    with pytest.raises(ValueError, match="captured for T = 37"):
        layer.forward_graph(g_part, x, lg)
    with pytest.raises(ValueError, match="not captured by this layer"):
        get_layer(TINY_MX, cuda_device).forward_graph(g_full, x, lg)


@pytest.mark.gpu
def test_layer_and_binding_refuse_bad_arguments(cuda_device):
    """Wrong sizes, dtypes, devices or strides raise on the host before any
    launch (the library takes raw pointers and cannot check them)."""
    wl = TINY
    layer = get_layer(wl, cuda_device)
    T, H, E = wl.T, wl.d_model, wl.num_experts
    x, lg = inputs.make_x(wl, seed=35).to(cuda_device), inputs.make_logits(wl, seed=36).to(cuda_device)
    big_x = torch.zeros(T + 1, H, dtype=torch.bfloat16, device=cuda_device)
    big_lg = torch.zeros(T + 1, E, dtype=torch.float32, device=cuda_device)
    with pytest.raises(ValueError, match="buffers hold"):
        layer.forward(big_x, big_lg)
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, lg.double())
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, lg[:, :E - 1].contiguous())
    with pytest.raises(ValueError, match="^x: "):
        layer.forward(x.float(), lg)
    with pytest.raises(ValueError, match="is on cpu"):
        layer.forward(x.cpu(), lg.cpu())
    with pytest.raises(ValueError, match="^logits: "):
        layer.forward(x, lg[:T - 1])
    with pytest.raises(ValueError, match="buffers hold"):
        layer.capture(T + 1)
    with pytest.raises(ValueError, match="not contiguous"):
        B.moe_permute(layer.cfg, T, torch.zeros(H, T, dtype=torch.bfloat16, device=cuda_device).t(),
                      layer.act_scale, layer.slot_to_row, layer.a_codes, layer.a_sf)
    with pytest.raises(ValueError, match="float32"):
        layer.quantize_experts(0, *(torch.zeros(1, 3, 3, device=cuda_device) for _ in range(3)))
    # the layer still works afterwards
    y = layer.forward(x, lg)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0 and y.shape == (T, H)


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX], ids=lambda w: w.name)
def test_host_pipeline_matches_eager(cuda_device, wl):
    """Five host batches through HostPipeline (uploads and downloads of
    neighbouring batches overlapping the layer) give, batch by batch, the
    eager results bit for bit."""
    from fp8_moe_expert_top_b200.layer import HostPipeline

    layer = get_layer(wl, cuda_device)
    n = 5
    xs = [inputs.make_x(wl, seed=40 + 2 * i).pin_memory() for i in range(n)]
    lgs = [inputs.make_logits(wl, seed=41 + 2 * i).pin_memory() for i in range(n)]
    ref = []
    for i in range(n):
        ref.append(layer.forward(xs[i].to(cuda_device), lgs[i].to(cuda_device)).cpu())
    pipe = HostPipeline(layer, wl.T)
    ys = [torch.full((wl.T, wl.d_model), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    pipe.run(xs, lgs, ys)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    for i in range(n):
        assert torch.equal(ys[i].view(torch.int16), ref[i].view(torch.int16)), i


@pytest.mark.gpu
def test_layer_stack_graph_matches_eager(cuda_device):
    """Three NVFP4 and two MXFP8 passes chained in one CUDA graph (each pass
    fed the previous one's output, fresh logits per pass) give the eager
    sequence's output bit for bit."""
    from fp8_moe_expert_top_b200.layer import capture_stack

    ln, lm = get_layer(TINY, cuda_device), get_layer(TINY_MX, cuda_device)
    T = TINY.T
    passes = [(ln if p < 3 else lm, inputs.make_logits(TINY, seed=60 + p).to(cuda_device)) for p in range(5)]
    x = inputs.make_x(TINY, seed=59).to(cuda_device)
    cur = x
    for layer, lg in passes:
        cur = layer.forward(cur, lg).clone()
    ref = cur.cpu()
    y_bufs = [torch.zeros(T, TINY.d_model, dtype=torch.bfloat16, device=cuda_device) for _ in range(2)]
    g, y = capture_stack(passes, x, y_bufs, T)
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.cpu().view(torch.int16), ref.view(torch.int16))
    assert int(ln.status.item()) == 0 and int(lm.status.item()) == 0


def _crafted_weights(wl, seed):
    """float32 weights of every expert, with crafted blocks in experts 0-3."""
    g = torch.Generator().manual_seed(seed)
    E, H, I = wl.num_experts, wl.d_model, wl.d_ffn
    wg = torch.randn(E, I, H, generator=g) / H ** 0.5
    wu = torch.randn(E, I, H, generator=g) / H ** 0.5
    wd = torch.randn(E, H, I, generator=g) / I ** 0.5
    wg[0].zero_()                                     # an all-zero matrix: tensor scale 1, zero codes
    wu[1].view(I, H // 16, 16)[:, ::2] = 0.0          # every other 16-element block all zero
    amax = wd[2].abs().max()                          # blocks whose maxima lie in [0.7, 1] of the
    mag = amax * (0.7 + 0.3 * torch.rand(8, I, generator=g))  # tensor max: the 4-candidate scale
    wd[2, :8, :] = mag * torch.sign(torch.randn(8, I, generator=g))  # saturates at 448
    wg[3, :, :16] = 0.25                              # a block of equal elements (tied errors)
    return wg.contiguous(), wu.contiguous(), wd.contiguous()


def _crafted_x(wl, seed):
    x = inputs.make_x(wl, seed=seed).float()
    x[0] = 0.0                                        # an all-zero token
    x[1, :16] = 0.0                                   # a zero block
    x[2] = 20.0 * torch.sign(x[2])                    # beyond the static scale's range: saturating codes
    x[3, 32:64] = x[3, 32:64] * 1e-30                 # values that round to zero codes
    return x.to(torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [TINY, TINY_MX], ids=lambda w: w.name)
def test_crafted_blocks(cuda_device, wl):
    """All-zero matrices and blocks, saturating 4-candidate scales, tied block
    errors, saturating and underflowing activations: weight codes, routing and
    activation codes bit-exact, the rest within the bars."""
    from fp8_moe_expert_top_b200.layer import ExpertLayer

    wg, wu, wd = _crafted_weights(wl, 70)
    layer = ExpertLayer(wl.num_experts, wl.top_k, wl.d_model, wl.d_ffn, wl.fmt, wl.T, cuda_device,
                        s_x=inputs.S_X, s_h=inputs.S_H, debug=True)
    layer.quantize_experts(0, wg.to(cuda_device), wu.to(cuda_device), wd.to(cuda_device))
    torch.cuda.synchronize()
    experts = {e: omoe.quantize_expert(wg[e].numpy(), wu[e].numpy(), wd[e].numpy(), wl.fmt)
               for e in range(wl.num_experts)}
    for e in range(4):
        assert_expert_equal(gpu_expert(layer, wl, e), experts[e], e)
    run_and_compare(layer, wl, _crafted_x(wl, 71), inputs.make_logits(wl, seed=72), experts)
