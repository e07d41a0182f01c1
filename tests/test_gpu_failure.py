"""Failure detection without a GPU fault (GPU).

Every wait in the library's kernels is bounded.  Here a wait that can never
complete (an mbarrier nothing arrives at) must give up after a short limit,
report through the device status word, and leave the context usable: the
next layer call still gives correct results.  Nothing in this file traps,
faults or hangs the GPU.
"""

import time

import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.moe_selftest_bounded_wait(status, 100_000_000)      # 100 ms limit
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status.item()) == B.MOE_DEVICE_TIMEOUT_SELFTEST
    assert 0.09 <= dt < 5.0, dt
    # the context still works: a small routing call after the timeout
    cfg = B.make_config(8, 2, 256, 128, "nvfp4")
    T = 16
    lg = torch.randn(T, 8, device=cuda_device)
    ids = torch.empty(T, 2, dtype=torch.int32, device=cuda_device)
    w = torch.empty(T, 2, device=cuda_device)
    cnt = torch.empty(8, dtype=torch.int32, device=cuda_device)
    off = torch.empty(9, dtype=torch.int32, device=cuda_device)
    R = B.moe_max_rows(cfg, T)
    ss = torch.empty(R, dtype=torch.int32, device=cuda_device)
    s2r = torch.empty(T * 2, dtype=torch.int32, device=cuda_device)
    ws = torch.empty(B.moe_route_workspace_bytes(cfg, T), dtype=torch.uint8, device=cuda_device)
    B.moe_route_topk(cfg, T, lg, ids, w, cnt, off, ss, s2r, ws)
    torch.cuda.synchronize()
    ref = torch.topk(lg, 2, dim=1).indices.to(torch.int32)
    assert torch.equal(ids, ref)
    assert int(cnt.sum().item()) == T * 2


def test_selftest_rejects_bad_limits():
    import ctypes
    fake = ctypes.c_void_p(0x10000)
    assert B.lib().moe_selftest_bounded_wait(fake, 10, None) == 1
    assert B.lib().moe_selftest_bounded_wait(None, 1_000_000, None) == 1
