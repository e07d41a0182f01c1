"""The routing entry point for callers that cannot allocate (GPU).

moe_route_topk_noalloc is meant for callers that hold only their input and
output buffers and cannot obtain scratch device memory; it routes with a
fixed scratch array inside the library instead of a caller workspace.  Its
results must equal moe_route_topk's bit for bit (routing is integer and
bit-exact work), on two calls in a row with different inputs, and a size
beyond its fixed scratch must be refused without running anything.  This
file sorts last so that a run stopping at its first failure has already run
every other test.
"""

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from fp8_moe_expert_top_b200 import inputs
from oracle import route as ort

SCRATCH_BYTES = 4 << 20


def _check_against_oracle(got, lg_cpu, T, E, k):
    """The no-allocation results equal the oracle's routing bit for bit."""
    r = ort.route(lg_cpu.numpy(), k, E)
    np.testing.assert_array_equal(got["ids"].cpu().numpy(), r["topk_ids"])
    np.testing.assert_array_equal(got["w"].cpu().numpy().view(np.uint32), r["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(got["counts"].cpu().numpy(), r["counts"])
    np.testing.assert_array_equal(got["offsets"].cpu().numpy(), r["offsets"])
    R = int(r["offsets"][-1])
    np.testing.assert_array_equal(got["sorted"][:R].cpu().numpy(), r["sorted_slots"])
    assert bool((got["sorted"][R:] == -1).all())
    np.testing.assert_array_equal(got["s2r"].cpu().numpy(), r["slot_to_row"])


def _buffers(cfg, T, E, k, dev):
    R = B.moe_max_rows(cfg, T)
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(ids=torch.full((T, k), -7, **i32), w=torch.full((T, k), -7.0, device=dev),
                counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
                sorted=torch.full((R,), -7, **i32), s2r=torch.full((T * k,), -7, **i32))


@pytest.mark.gpu
def test_route_noalloc_matches_route_on_two_calls(cuda_device):
    dev = cuda_device
    wl = inputs.WORKLOADS["prefill_nvfp4_skewed"]
    E, k = wl.num_experts, wl.top_k
    cfg = B.make_config(E, k, wl.d_model, wl.d_ffn, wl.fmt)
    for call, T in enumerate([4096, 64]):
        lg = inputs.make_logits(wl, T=T, seed=1000 + call).to(dev)
        ref = _buffers(cfg, T, E, k, dev)
        got = _buffers(cfg, T, E, k, dev)
        ws = torch.empty(B.moe_route_workspace_bytes(cfg, T), dtype=torch.uint8, device=dev)
        B.moe_route_topk(cfg, T, lg, ref["ids"], ref["w"], ref["counts"], ref["offsets"], ref["sorted"], ref["s2r"],
                         ws)
        B.moe_route_topk_noalloc(cfg, T, lg, got["ids"], got["w"], got["counts"], got["offsets"], got["sorted"],
                                 got["s2r"])
        torch.cuda.synchronize()
        for name in ref:
            a = ref[name].cpu().numpy()
            b = got[name].cpu().numpy()
            np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32), err_msg=f"call {call}: {name}")
        counts = got["counts"].cpu().numpy().astype(np.int64)
        assert int(got["offsets"][-1].item()) == int(((counts + 127) // 128 * 128).sum())
        _check_against_oracle(got, lg.cpu(), T, E, k)


@pytest.mark.gpu
def test_route_noalloc_at_its_size_limit(cuda_device):
    """The largest batch the fixed scratch holds (43,680 tokens at 384
    experts: 4 MiB of bitmaps and counts) routes like moe_route_topk and the
    oracle; one token more is refused."""
    dev = cuda_device
    wl = inputs.WORKLOADS["prefill_nvfp4_skewed"]
    E, k = wl.num_experts, wl.top_k
    cfg = B.make_config(E, k, wl.d_model, wl.d_ffn, wl.fmt)
    T = 43680
    assert B.moe_route_workspace_bytes(cfg, T) <= SCRATCH_BYTES < B.moe_route_workspace_bytes(cfg, T + 1)
    lg_cpu = inputs.make_logits(wl, T=T, seed=2024)
    lg = lg_cpu.to(dev)
    ref = _buffers(cfg, T, E, k, dev)
    got = _buffers(cfg, T, E, k, dev)
    ws = torch.empty(B.moe_route_workspace_bytes(cfg, T), dtype=torch.uint8, device=dev)
    B.moe_route_topk(cfg, T, lg, ref["ids"], ref["w"], ref["counts"], ref["offsets"], ref["sorted"], ref["s2r"], ws)
    B.moe_route_topk_noalloc(cfg, T, lg, got["ids"], got["w"], got["counts"], got["offsets"], got["sorted"],
                             got["s2r"])
    torch.cuda.synchronize()
    for name in ref:
        np.testing.assert_array_equal(ref[name].cpu().numpy().view(np.uint32), got[name].cpu().numpy().view(np.uint32),
                                      err_msg=name)
    _check_against_oracle(got, lg_cpu, T, E, k)
    over = _buffers(cfg, T + 1, E, k, dev)
    lg1 = torch.zeros(T + 1, E, dtype=torch.float32, device=dev)
    with pytest.raises(B.MoeError) as ei:
        B.moe_route_topk_noalloc(cfg, T + 1, lg1, over["ids"], over["w"], over["counts"], over["offsets"],
                                 over["sorted"], over["s2r"])
    assert ei.value.status == 3           # MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((over["ids"] == -7).all()) and bool((over["sorted"] == -7).all())  # nothing was enqueued


@pytest.mark.gpu
def test_route_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    cfg = B.make_config(1024, 8, 256, 128, "nvfp4")
    T = 1 << 18                           # needs far more than the fixed 4 MiB of scratch
    assert B.moe_route_workspace_bytes(cfg, T) > (4 << 20)
    fake = torch.empty(16, dtype=torch.int32, device=cuda_device)
    with pytest.raises(B.MoeError) as ei:
        B.moe_route_topk_noalloc(cfg, T, fake, fake, fake, fake, fake, fake, fake)
    assert ei.value.status == 3           # MOE_ERR_WORKSPACE
