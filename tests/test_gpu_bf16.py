"""BF16 experts with LoRA adapters (GPU).

Pages "thinkingmachines/Inkling-2-Small" (Configurations) and "Thinking
Machines releases Inkling 2 Small weights under Apache 2.0" ("LoRA and
reinforcement learning"): adapters on the routed experts need BF16 expert
weights.  The library folds each adapter's expand step into the expert GEMM
as one extra 64-element K tile (z = s A a in the rows, B in the weights) and
computes z on the tensor cores (the shrink), rounded to bf16.

  * exact: grid-valued bf16 weights and rows, adapter A with two non-zeros
    per row of +-1/8 (so every z is exact in bf16) and B on a grid: the
    gate/up outputs must equal the exact float64 values bit for bit, the h
    shrink must equal bf16(s * (A_down h)) of the kernel's own h (up to one
    bf16 ulp where the float32 sum of its two products rounds), and the down
    output (given h and its adapter tile) bf16 of the exact sum;
  * parity with the oracle (oracle.moe.forward_bf16) on seeded layers, tiny
    and at d_model 4096 / ffn 2560 / 384 experts: routing bit-exact; gate/up
    within the bound of the float32 sums and of the bf16 rounding of z,
        |g - g_ref| <= H 2^-23 sum|a w| + sum_j dz_j |B_j| + 2^-22 sum_j |z_j B_j|,
        dz_j = 2^-9 |z_j| + s H 2^-22 sum_h |a_h A_jh|;
    h (bf16) within relative Frobenius 2^-7 (two independent bf16 roundings
    of values that already differ by that bound); y within 1e-2.
"""

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from fp8_moe_expert_top_b200 import inputs
from fp8_moe_expert_top_b200.layer import ExpertLayer
from oracle import formats as ofm
from oracle import moe as omoe
from oracle import route as ort

from helpers import ACT_TR, rel_fro, tile_matrix, tile_offsets

S = inputs.LORA_SCALING


def _bf16_bytes(a):
    """[rows, K] float (bf16 values) -> [rows, 2K] bytes of bf16."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.uint8).numpy().reshape(a.shape[0], -1)


def _grid(rng, shape, step, lim):
    n = int(round(lim / step))
    return (rng.integers(-n, n + 1, shape) * step).astype(np.float32)


def _sparse_a(rng, r, K):
    a = np.zeros((r, K), dtype=np.float32)
    for j in range(r):
        idx = rng.choice(K, 2, replace=False)
        a[j, idx] = rng.choice([-0.125, 0.125], 2)
    return a


def _bf(x, dev):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(dev)


@pytest.mark.gpu
@pytest.mark.parametrize("H,I", [(256, 128), (1024, 384)])
def test_bf16_adapter_gemms_exact(cuda_device, H, I):
    dev = cuda_device
    rng = np.random.default_rng(H + I)
    counts = np.array([200, 0, 130], dtype=np.int32)
    E, k, r = len(counts), 1, 32
    T = int(counts.sum())
    offsets = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
    cfg = B.make_config(E, k, H, I, "bf16")
    R = B.moe_max_rows(cfg, T)
    W = {e: {"gate": _grid(rng, (I, H), 0.125, 0.25), "up": _grid(rng, (I, H), 0.125, 0.25),
             "down": _grid(rng, (H, I), 0.125, 0.25)} for e in range(E)}
    L = {e: {"gate": (_sparse_a(rng, r, H), _grid(rng, (I, r), 0.25, 1.0)),
             "up": (_sparse_a(rng, r, H), _grid(rng, (I, r), 0.25, 1.0)),
             "down": (_sparse_a(rng, r, I), _grid(rng, (H, r), 0.25, 1.0))} for e in range(E)}
    layout = B.moe_get_weights_layout(cfg)
    packed = torch.zeros(layout.total_bytes, dtype=torch.uint8, device=dev)
    st = lambda m: torch.stack([_bf(W[e][m], dev) for e in range(E)]).contiguous()            # noqa: E731
    lo = lambda m, i: torch.stack([_bf(L[e][m][i], dev) for e in range(E)]).contiguous()      # noqa: E731
    B.moe_pack_weights_bf16(cfg, 0, E, st("gate"), st("up"), st("down"),
                            (lo("gate", 0), lo("gate", 1), lo("up", 0), lo("up", 1), lo("down", 0), lo("down", 1)),
                            r, S, packed)
    # rows of A: grid values in the rows in use, random bytes (NaN included) in padding rows
    kbA = 2 * H + 128
    a_raw = rng.integers(0, 256, (R, kbA), dtype=np.uint8)
    A = np.zeros((R, H))
    for e in range(E):
        lo_, c = offsets[e], counts[e]
        if c:
            vals = _grid(rng, (c, H), 0.25, 2.0)
            a_raw[lo_:lo_ + c, :2 * H] = _bf16_bytes(vals)
            A[lo_:lo_ + c] = vals
    d_a = torch.from_numpy(tile_matrix(a_raw, ACT_TR)).to(dev)
    d_off = torch.from_numpy(offsets).to(dev)
    d_cnt = torch.from_numpy(counts).to(dev)
    h_codes = torch.zeros(B.moe_codes_bytes(cfg, R, I), dtype=torch.uint8, device=dev)
    dbg = torch.full((R, 2 * I), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B.moe_forward_gateup(cfg, T, packed, d_a, None, None, None, d_off, d_cnt, h_codes, None, dbg, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = dbg.cpu().numpy()
    for e in range(E):
        lo_, c = offsets[e], counts[e]
        if not c:
            continue
        a = A[lo_:lo_ + c]
        for m, cols in (("gate", slice(0, I)), ("up", slice(I, 2 * I))):
            ref = omoe.lora_project(a, W[e][m], L[e][m][0], L[e][m][1], S)
            np.testing.assert_array_equal(got[lo_:lo_ + c, cols], ref.astype(np.float32), err_msg=f"{m} e={e}")
    # the shrink of h: bf16(s * (A_down h)) of the kernel's own h, in h's adapter tile
    kbH = 2 * I + 128
    rows_in_use = np.concatenate([np.arange(offsets[e], offsets[e] + counts[e]) for e in range(E)])
    hb = h_codes.cpu().numpy().reshape(-1)[tile_offsets(rows_in_use, kbH, ACT_TR)]
    hv = torch.from_numpy(np.ascontiguousarray(hb[:, :2 * I])).view(torch.bfloat16).float().numpy().astype(np.float64)
    zv = torch.from_numpy(np.ascontiguousarray(hb[:, 2 * I:2 * I + 128])).view(torch.bfloat16).float().numpy()
    i0 = 0
    for e in range(E):
        c = counts[e]
        if not c:
            continue
        z_ref = ofm.bf16_round(S * (hv[i0:i0 + c] @ L[e]["down"][0].astype(np.float64).T))
        # two products per z: exact in float32 unless their exponents lie far
        # apart, where one float32 rounding may move the bf16 result by an ulp
        diff = zv[i0:i0 + c, :32] != z_ref
        assert diff.mean() <= 1e-3, (e, diff.mean())
        np.testing.assert_allclose(zv[i0:i0 + c, :32], z_ref, rtol=2.0 ** -7, atol=0, err_msg=f"h shrink e={e}")
        assert np.all(zv[i0:i0 + c, 32:] == 0)
        i0 += c
    # down over a given h and its adapter tile
    h_raw = rng.integers(0, 256, (R, kbH), dtype=np.uint8)
    Hm = np.zeros((R, I))
    for e in range(E):
        lo_, c = offsets[e], counts[e]
        if c:
            hv = _grid(rng, (c, I), 0.25, 2.0)
            z = S * (hv.astype(np.float64) @ L[e]["down"][0].astype(np.float64).T)   # exact in bf16
            h_raw[lo_:lo_ + c, :2 * I] = _bf16_bytes(hv)
            h_raw[lo_:lo_ + c, 2 * I:] = _bf16_bytes(np.concatenate([z, np.zeros((c, 32))], axis=1))
            Hm[lo_:lo_ + c] = hv
    out = torch.full((R, H), float("nan"), dtype=torch.bfloat16, device=dev)
    B.moe_forward_down(cfg, T, packed, torch.from_numpy(tile_matrix(h_raw, ACT_TR)).to(dev), None, None, d_off,
                       d_cnt, out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o = out.float().cpu().numpy().astype(np.float64)
    for e in range(E):
        lo_, c = offsets[e], counts[e]
        if c:
            ref = ofm.bf16_round(omoe.lora_project(Hm[lo_:lo_ + c], W[e]["down"], L[e]["down"][0], L[e]["down"][1], S))
            np.testing.assert_array_equal(o[lo_:lo_ + c], ref, err_msg=f"down e={e}")


def _bf16_layer(wl, dev, lora=True, debug=True, T=None):
    T = wl.T if T is None else T
    layer = ExpertLayer(wl.num_experts, wl.top_k, wl.d_model, wl.d_ffn, wl.fmt, T, dev, debug=debug)
    chunk = 16
    for e0 in range(0, wl.num_experts, chunk):
        n = min(chunk, wl.num_experts - e0)
        ws = [inputs.make_expert_weights_bf16(wl, e, device=dev) for e in range(e0, e0 + n)]
        w3 = [torch.stack([w[m] for w in ws]).contiguous() for m in range(3)]
        lo = None
        if lora:
            ls = [inputs.make_expert_lora(wl, e, device=dev) for e in range(e0, e0 + n)]
            lo = tuple(torch.stack([l_[m] for l_ in ls]).contiguous() for m in range(6))
        layer.pack_experts_bf16(e0, *w3, lora=lo, lora_rank=inputs.LORA_RANK, lora_scaling=S)
    torch.cuda.synchronize()
    return layer


def _oracle_expert(wl, e, lora, dev):
    """The oracle's copy of expert e: drawn on the layer's device (the same
    generator), as float arrays."""
    w = {m: t.float().cpu().numpy() for m, t in zip(("gate", "up", "down"),
                                                    inputs.make_expert_weights_bf16(wl, e, device=dev))}
    lo = None
    if lora:
        t = [x.float().cpu().numpy() for x in inputs.make_expert_lora(wl, e, device=dev)]
        lo = {"gate": (t[0], t[1]), "up": (t[2], t[3]), "down": (t[4], t[5])}
    return w, lo


@pytest.mark.gpu
@pytest.mark.parametrize("name,lora", [("tiny_bf16_lora", True), ("tiny_bf16_lora", False),
                                       ("decode_bf16_lora", True)])
def test_bf16_layer_against_oracle(cuda_device, name, lora):
    """Every token of the tiny layer; tokens 0, T/2 and T-1 at full size (the
    oracle needs float copies of each expert those tokens select)."""
    dev = cuda_device
    wl = inputs.WORKLOADS[name]
    layer = _bf16_layer(wl, dev, lora=lora)
    x, lg = inputs.make_x(wl), inputs.make_logits(wl)
    y = layer.forward(x.to(dev), lg.to(dev))
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    T, k, E, H, I = wl.T, wl.top_k, wl.num_experts, wl.d_model, wl.d_ffn
    r = ort.route(lg.numpy(), k, E)
    np.testing.assert_array_equal(layer.topk_ids.cpu().numpy(), r["topk_ids"])
    np.testing.assert_array_equal(layer.expert_offsets.cpu().numpy(), r["offsets"])
    sample = list(range(T)) if wl.d_model <= 256 else [0, T // 2, T - 1]
    need = sorted(set(int(e) for t in sample for e in r["topk_ids"][t]))
    ws, los = {}, {}
    for e in need:
        ws[e], los[e] = _oracle_expert(wl, e, lora, dev)
    xs = x[sample].float().numpy()
    ref = omoe.forward_bf16(xs, lg[sample].numpy(), ws, {e: l for e, l in los.items() if l is not None}, k, S, E)
    # rows of the sampled tokens on both sides
    gpu_rows = np.array([int(r["slot_to_row"][t * k + j]) for t in sample for j in range(k)])
    ref_rows = np.array([int(ref["slot_to_row"][i * k + j]) for i in range(len(sample)) for j in range(k)])
    experts = np.array([int(r["topk_ids"][t, j]) for t in sample for j in range(k)])
    a = np.repeat(xs.astype(np.float64), k, axis=0)
    dbg = layer.gateup_debug.index_select(0, torch.as_tensor(gpu_rows, device=dev)).cpu().numpy().astype(np.float64)
    worst = 0.0
    for m, cols in (("gate", slice(0, I)), ("up", slice(I, 2 * I))):
        g_ref = ref[m][ref_rows]
        err = np.abs(dbg[:, cols] - g_ref)
        for i, e in enumerate(experts):
            bound = H * 2.0 ** -23 * (np.abs(a[i]) @ np.abs(ws[e][m]).T)
            if los[e] is not None:
                la, lb = los[e][m][0].astype(np.float64), np.abs(los[e][m][1]).astype(np.float64)
                z = S * (a[i] @ la.T)
                # z on the GPU: a float32 sum over H products, then one bf16 rounding
                dz = 2.0 ** -9 * np.abs(z) + S * H * 2.0 ** -22 * (np.abs(a[i]) @ np.abs(la).T)
                bound = bound + dz @ lb.T + 2.0 ** -22 * (np.abs(z) @ lb.T)
            assert np.all(err[i] <= bound + 1e-30), (e, m, float(np.max(err[i] - bound)))
        worst = max(worst, rel_fro(dbg[:, cols], g_ref))
    # h: bf16 in the tiled layout
    kbH = 2 * I + 128
    off = torch.as_tensor(tile_offsets(gpu_rows, kbH, ACT_TR)[:, :2 * I].reshape(-1), device=dev)
    hb = layer.h_codes.reshape(-1).index_select(0, off).cpu().view(torch.bfloat16).float().numpy()
    err_h = rel_fro(hb.reshape(len(gpu_rows), I), ref["h"][ref_rows])
    assert err_h <= 2.0 ** -7, err_h
    err_y = rel_fro(y.float().cpu().numpy()[sample], ref["y"])
    print(f"{name} lora={lora}: gate/up {worst:.2e} h {err_h:.2e} y {err_y:.2e}")
    assert err_y <= 1e-2, err_y


@pytest.mark.gpu
def test_bf16_graph_replay_matches_eager(cuda_device):
    dev = cuda_device
    wl = inputs.WORKLOADS["tiny_bf16_lora"]
    layer = _bf16_layer(wl, dev, debug=False)
    x, lg = inputs.make_x(wl).to(dev), inputs.make_logits(wl).to(dev)
    y_eager = layer.forward(x, lg).clone()
    g = layer.capture(wl.T)
    y_graph = layer.forward_graph(g, x, lg).clone()
    torch.cuda.synchronize()
    assert torch.equal(y_eager, y_graph)
