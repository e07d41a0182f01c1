"""Router scores fused with the top-k, against the oracle (GPU).

moe_router_topk computes logits = x W_r^T on the tensor cores (bf16
products, float32 accumulation in the tensor core's order) and reduces them
to the top-k in the same kernel.  The oracle sums the same bf16 products in
float64 and rounds once (oracle.route.router_logits).

  * Grid-valued x and W_r (multiples of 1/4 and 1/8 of magnitude <= 2 and
    <= 1/4): every product is a multiple of 1/32 and every partial sum stays
    below 2^11, so any summation order gives the exact sum in float32.  The
    scores (debug copy) and the whole routing (ids, softmax weights as bits,
    counts, offsets, slot sort) must then equal the oracle's bit for bit.
    Grid values tie often, which also exercises the lower-index tie rule.
  * Random x ~ N(0, 1) and W_r ~ N(0, 1/H) in bf16: each score is within the
    order-independent float32 summation bound of the exact sum,
        |s - exact| <= (H * 2^-23) * sum_h |x_h w_h| + 2^-24 |exact|
    (H additions, each off by at most one float32 ulp even if the hardware
    truncates, and the final rounding),
    and on every token whose k+1 largest exact scores are separated by more
    than twice the largest distance of its scores from the exact sums (the
    kernel's, bounded as above, plus the oracle's half-ulp rounding) the
    selection and its order are unique on both sides: ids must
    equal the oracle's, and each weight is within the first-order effect of
    its token's score differences (twice the largest, plus float32 roundings).  For every
    token the routing must be consistent: counts, padded offsets and the slot
    sort describe the kernel's own selection.
"""

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from oracle import route as ort

# (T, E, H, k): tiny, one token, a ragged batch at the model's size, experts
# not a multiple of 128, the 512-expert limit (two-stage ring), several tiles.
# Batches of up to 37 row tiles split K over clusters of 4 or 8 CTAs (the
# first four cases and 777 tokens: 8; 64 and 129 tokens at d_model 256: 4).
# Up to 74 row tiles with E a multiple of 128 split the experts over a
# two-CTA cluster: the 512-expert case (2 tiles), 5000 tokens (40 tiles, 384,
# 256 and 128 experts) and 4900 tokens at 512 experts.  9600 tokens (75 tiles)
# take the one-CTA-per-tile kernel, at 384 and at 512 experts (two-stage ring).
GRID_CASES = [(64, 8, 256, 2), (1, 384, 4096, 8), (777, 384, 4096, 8), (300, 200, 512, 6), (256, 512, 1024, 8),
              (129, 128, 256, 1), (9600, 384, 512, 8), (5000, 384, 512, 8), (5000, 256, 512, 4),
              (5000, 128, 256, 2), (4900, 512, 1024, 8), (9600, 512, 256, 8)]


def _bufs(cfg, T, E, k, dev):
    R = B.moe_max_rows(cfg, T)
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(ids=torch.full((max(T, 1), k), -7, **i32), w=torch.full((max(T, 1), k), -7.0, device=dev),
                counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
                sorted=torch.full((R,), -7, **i32), s2r=torch.full((max(T * k, 1),), -7, **i32),
                ws=torch.empty(B.moe_route_workspace_bytes(cfg, T), dtype=torch.uint8, device=dev),
                status=torch.zeros(1, **i32))


def _run(cfg, T, x, w, b, logits=None):
    B.moe_router_topk(cfg, T, x, w, logits, b["ids"], b["w"], b["counts"], b["offsets"], b["sorted"], b["s2r"], b["ws"],
                      b["status"])


def _grid(rng, shape, step, lim):
    n = int(round(lim / step))
    return (rng.integers(-n, n + 1, shape) * step).astype(np.float32)


def _check_routing_equal(b, r, T):
    np.testing.assert_array_equal(b["ids"][:T].cpu().numpy(), r["topk_ids"])
    np.testing.assert_array_equal(b["w"][:T].cpu().numpy().view(np.uint32), r["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(b["counts"].cpu().numpy(), r["counts"])
    np.testing.assert_array_equal(b["offsets"].cpu().numpy(), r["offsets"])
    R = int(r["offsets"][-1])
    np.testing.assert_array_equal(b["sorted"][:R].cpu().numpy(), r["sorted_slots"])
    assert bool((b["sorted"][R:] == -1).all())
    np.testing.assert_array_equal(b["s2r"][:T * r["topk_ids"].shape[1]].cpu().numpy(), r["slot_to_row"])


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,H,k", GRID_CASES)
def test_router_grid_values_bit_exact(cuda_device, T, E, H, k):
    dev = cuda_device
    rng = np.random.default_rng(T * 31 + E + H + k)
    x = _grid(rng, (T, H), 0.25, 2.0)
    w = _grid(rng, (E, H), 0.125, 0.25)
    cfg = B.make_config(E, k, H, 128, "nvfp4")
    xd = torch.from_numpy(x).to(torch.bfloat16).to(dev)
    wd = torch.from_numpy(w).to(torch.bfloat16).to(dev)
    assert torch.equal(xd.float().cpu(), torch.from_numpy(x)) and torch.equal(wd.float().cpu(), torch.from_numpy(w))
    b = _bufs(cfg, T, E, k, dev)
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device=dev)
    _run(cfg, T, xd, wd, b, logits)
    b2 = _bufs(cfg, T, E, k, dev)
    _run(cfg, T, xd, wd, b2)                      # without the debug copy of the scores
    torch.cuda.synchronize()
    assert int(b["status"].item()) == 0 and int(b2["status"].item()) == 0
    ref_logits = ort.router_logits(x, w)
    np.testing.assert_array_equal(logits.cpu().numpy(), ref_logits)
    r = ort.router_route(x, w, k, E)
    _check_routing_equal(b, r, T)
    _check_routing_equal(b2, r, T)


def _check_consistent(b, T, E, k):
    """counts / offsets / slot sort describe the kernel's own selection."""
    ids = b["ids"][:T].cpu().numpy().astype(np.int64)
    assert ids.min() >= 0 and ids.max() < E
    assert all(len(set(row)) == k for row in ids.tolist())
    counts = np.bincount(ids.reshape(-1), minlength=E)
    np.testing.assert_array_equal(b["counts"].cpu().numpy(), counts)
    offsets = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)])
    np.testing.assert_array_equal(b["offsets"].cpu().numpy(), offsets)
    srt = b["sorted"].cpu().numpy().astype(np.int64)
    s2r = b["s2r"][:T * k].cpu().numpy().astype(np.int64)
    for e in range(E):
        seg = srt[offsets[e]:offsets[e] + counts[e]]
        assert np.all(ids.reshape(-1)[seg] == e) and np.all(np.diff(seg // k) > 0)
        assert np.all(srt[offsets[e] + counts[e]:offsets[e + 1]] == -1)
    np.testing.assert_array_equal(srt[s2r], np.arange(T * k))


@pytest.mark.gpu
@pytest.mark.parametrize("T", [64, 2048, 8192, 16384])
def test_router_random_inputs_within_bound(cuda_device, T):
    dev = cuda_device
    E, H, k = 384, 4096, 8
    g = torch.Generator().manual_seed(T)
    xd = torch.randn(T, H, generator=g).to(torch.bfloat16)
    wd = (torch.randn(E, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    x, w = xd.float().numpy(), wd.float().numpy()
    cfg = B.make_config(E, k, H, 2560, "nvfp4")
    b = _bufs(cfg, T, E, k, dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    _run(cfg, T, xd.to(dev), wd.to(dev), b, logits)
    torch.cuda.synchronize()
    assert int(b["status"].item()) == 0
    got = logits.cpu().numpy().astype(np.float64)
    exact = x.astype(np.float64) @ w.astype(np.float64).T          # within float64 rounding of the exact sums
    mag = np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T
    bound = H * 2.0 ** -23 * mag + np.abs(exact) * 2.0 ** -24
    assert np.all(np.abs(got - exact) <= bound), float(np.max(np.abs(got - exact) / bound))
    ref = ort.router_route(x, w, k, E)
    # Tokens whose top k+1 exact scores are separated by more than twice the
    # largest distance of any of the token's scores from the exact sum, on
    # either side (the kernel's, now bounded above, and the oracle's float32
    # rounding, at most half an ulp): there both orders equal the exact one.
    dev_t = (np.max(np.abs(got - exact), axis=1, keepdims=True)
             + np.max(np.abs(exact), axis=1, keepdims=True) * 2.0 ** -24)
    srt = -np.sort(-exact, axis=1)[:, :k + 1]
    unique = np.all(srt[:, :-1] - srt[:, 1:] > 2.0 * dev_t, axis=1)
    assert unique.mean() >= 0.5, unique.mean()
    ids = b["ids"].cpu().numpy()
    np.testing.assert_array_equal(ids[unique], ref["topk_ids"][unique])
    # softmax weights: d(log w_j) = dl_j - sum_i w_i dl_i, so a weight moves
    # by at most about twice the largest score difference of its token (plus
    # a few float32 roundings in exp, the sum and the division)
    ref_logits = ort.router_logits(x, w).astype(np.float64)
    sel = ref["topk_ids"].astype(np.int64)
    dl = np.max(np.abs(np.take_along_axis(got, sel, 1) - np.take_along_axis(ref_logits, sel, 1)), axis=1)
    wg = b["w"].cpu().numpy().astype(np.float64)
    wr = ref["topk_w"].astype(np.float64)
    rel = np.abs(wg - wr) / wr
    tol = 2.1 * dl[:, None] + 1e-6
    assert np.all(rel[unique] <= tol[unique]), float(np.max(rel[unique] - tol[unique]))
    _check_consistent(b, T, E, k)


@pytest.mark.gpu
def test_router_empty_batch(cuda_device):
    dev = cuda_device
    cfg = B.make_config(384, 8, 4096, 2560, "nvfp4")
    b = _bufs(cfg, 0, 384, 8, dev)
    x = torch.zeros(1, 4096, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(384, 4096, dtype=torch.bfloat16, device=dev)
    _run(cfg, 0, x, w, b)
    torch.cuda.synchronize()
    assert bool((b["counts"] == 0).all()) and bool((b["offsets"] == 0).all())


@pytest.mark.gpu
def test_router_refuses_more_than_512_experts(cuda_device):
    dev = cuda_device
    cfg = B.make_config(640, 8, 256, 128, "nvfp4")
    b = _bufs(cfg, 4, 640, 8, dev)
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(640, 256, dtype=torch.bfloat16, device=dev)
    with pytest.raises(B.MoeError) as ei:
        _run(cfg, 4, x, w, b)
    assert ei.value.status == 2            # MOE_ERR_UNSUPPORTED
