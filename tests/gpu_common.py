"""Shared pieces of the GPU parity tests: building a layer on the device,
quantizing seeded weights, and running the oracle on the same inputs."""

import numpy as np
import torch

from fp8_moe_expert_top_b200 import inputs
from fp8_moe_expert_top_b200.layer import ExpertLayer
from oracle import moe as omoe

from helpers import decode_expert


def build_layer(wl, device, T=None, debug=True, weight_device=None, chunk=32):
    """ExpertLayer for workload wl with every expert's seeded weights quantized."""
    T = wl.T if T is None else T
    layer = ExpertLayer(wl.num_experts, wl.top_k, wl.d_model, wl.d_ffn, wl.fmt, T, device,
                        s_x=inputs.S_X, s_h=inputs.S_H, debug=debug)
    wdev = weight_device or ("cpu" if wl.d_model * wl.d_ffn * wl.num_experts <= (1 << 24) else device)
    for e0 in range(0, wl.num_experts, chunk):
        n = min(chunk, wl.num_experts - e0)
        ws = [inputs.make_expert_weights(wl, e, device=wdev) for e in range(e0, e0 + n)]
        wg = torch.stack([w[0] for w in ws]).to(device).contiguous()
        wu = torch.stack([w[1] for w in ws]).to(device).contiguous()
        wd = torch.stack([w[2] for w in ws]).to(device).contiguous()
        layer.quantize_experts(e0, wg, wu, wd)
        del ws, wg, wu, wd
    torch.cuda.synchronize()
    layer.weight_device = wdev
    return layer


def oracle_expert(wl, e, device):
    """The oracle's own quantization of expert e's float32 weights."""
    wg, wu, wd = (w.cpu().numpy() for w in inputs.make_expert_weights(wl, e, device=device))
    return omoe.quantize_expert(wg, wu, wd, wl.fmt)


def gpu_expert(layer, wl, e):
    """Expert e's (codes, scales, tensor scale) read back from the device,
    copying only that expert's byte ranges of the packed buffer."""
    get = lambda off, n: layer.packed[off:off + n].cpu().numpy()  # noqa: E731
    return decode_expert(get, layer.layout, wl.fmt, e, wl.d_model, wl.d_ffn)


def assert_expert_equal(got, ref, e):
    for m in ("gate", "up", "down"):
        gc, gs, gt = got[m]
        rc, rs, rt = ref[m]
        assert np.float32(gt) == np.float32(rt), (e, m, gt, rt)
        nbad_c = int(np.sum(gc != rc))
        nbad_s = int(np.sum(gs != rs))
        assert nbad_c == 0 and nbad_s == 0, (e, m, nbad_c, nbad_s)
