"""GPU parity at the full sizes of the named layers (GPU).

Layers (d_model 4096, expert ffn 2560, 384 experts, top-8): decode NVFP4
(T = 64), decode MXFP8 (T = 256), prefill NVFP4 (T = 8192), prefill NVFP4
with Zipf-skewed routing (T = 16384) and prefill MXFP8 (T = 8192), run with
the same ExpertLayer the benchmark times.  Checked against the oracle:
  * routing of every token: top-k ids, softmax weights, counts, offsets and
    the slot permutation, bit-exact;
  * on sampled tokens (the oracle is too slow for all of them): the weight
    codes of every expert they select, their activation codes (bit-exact),
    their gate/up rows (relative Frobenius error <= 1e-4), their requantized
    intermediate (at most 1e-3 of (code, block scale) pairs differ) and
    their bf16 output (relative Frobenius error <= 1e-2);
  * on every token: a finite output.
"""

import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import inputs
from oracle import formats as ofm
from oracle import moe as omoe
from oracle import route as ort

from gpu_common import assert_expert_equal, build_layer, gpu_expert
from helpers import ACT_TR, kb_padded, rel_fro, sfvec, sf_index, tile_offsets, unpack_codes

FULL = ["decode_nvfp4", "decode_mxfp8", "prefill_nvfp4", "prefill_nvfp4_skewed", "prefill_mxfp8"]


def _quantize_job(job):
    e, fmt, wg, wu, wd = job
    return e, omoe.quantize_expert(wg, wu, wd, fmt)


def oracle_experts(wl, experts, device):
    jobs = []
    for e in experts:
        wg, wu, wd = (w.cpu().numpy() for w in inputs.make_expert_weights(wl, e, device=device))
        jobs.append((e, wl.fmt, wg, wu, wd))
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(len(jobs), max(1, os.cpu_count() or 1))) as pool:
        return dict(pool.map(_quantize_job, jobs))


def rows_np(t, rows):
    idx = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=t.device)
    return t.index_select(0, idx).cpu().numpy()


def tiled_rows(t, rows, K, fmt):
    """Codes [len(rows), K] of the given rows of a tiled device code buffer."""
    kb = kb_padded(K, fmt)
    off = torch.as_tensor(tile_offsets(rows, kb, ACT_TR).reshape(-1), device=t.device)
    raw = t.reshape(-1).index_select(0, off).cpu().numpy().reshape(len(rows), kb)
    return unpack_codes(fmt, raw, len(rows), K)


@pytest.mark.gpu
@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(cuda_device, name):
    wl = inputs.WORKLOADS[name]
    dev = cuda_device
    layer = build_layer(wl, dev, debug=True, weight_device=dev)
    x, lg = inputs.make_x(wl), inputs.make_logits(wl)
    layer.status.zero_()
    y = layer.forward(x.to(dev), lg.to(dev))
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    T, k, E, H, I, v = wl.T, wl.top_k, wl.num_experts, wl.d_model, wl.d_ffn, sfvec(wl.fmt)

    # routing of every token
    r = ort.route(lg.numpy(), k, E)
    np.testing.assert_array_equal(layer.topk_ids.cpu().numpy(), r["topk_ids"])
    np.testing.assert_array_equal(layer.topk_w.cpu().numpy().view(np.uint32), r["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(layer.expert_counts.cpu().numpy(), r["counts"])
    np.testing.assert_array_equal(layer.expert_offsets.cpu().numpy(), r["offsets"])
    R = int(r["offsets"][-1])
    np.testing.assert_array_equal(layer.sorted_slots[:R].cpu().numpy(), r["sorted_slots"])
    np.testing.assert_array_equal(layer.slot_to_row.cpu().numpy(), r["slot_to_row"])
    yall = y.float().cpu().numpy()
    assert np.all(np.isfinite(yall))

    # sampled tokens
    rng = np.random.default_rng(T)
    sample = sorted(set([0, T - 1] + [int(t) for t in rng.integers(0, T, 1)]))[:2]
    need = sorted(set(int(e) for t in sample for e in r["topk_ids"][t]))
    oq = oracle_experts(wl, need, dev)
    for e in need:
        assert_expert_equal(gpu_expert(layer, wl, e), oq[e], e)

    xs = x[sample].float().numpy()
    ref = omoe.forward_tokens(xs, lg[sample].numpy(), oq, k, wl.fmt, inputs.S_X, inputs.S_H)
    rows = [int(r["slot_to_row"][t * k + j]) for t in sample for j in range(k)]
    # activation codes of the sampled rows
    a_codes = tiled_rows(layer.a_codes, rows, H, wl.fmt)
    a_sf_all = layer.a_sf.cpu().numpy()
    sfi = sf_index(layer.R_max, H // v)
    a_sf = a_sf_all[sfi[rows]]
    for i, t in enumerate(sample):
        for j in range(k):
            np.testing.assert_array_equal(a_codes[i * k + j], ref["a_codes"][i])
            np.testing.assert_array_equal(a_sf[i * k + j], ref["a_sf"][i])
    # gate/up and the intermediate on the sampled rows
    dbg = rows_np(layer.gateup_debug, rows)
    h_codes = tiled_rows(layer.h_codes, rows, I, wl.fmt)
    h_sf = layer.h_sf.cpu().numpy()[sf_index(layer.R_max, I // v)[rows]]
    a_deq = omoe.dequantize_rows(ref["a_codes"], ref["a_sf"], wl.fmt, inputs.S_X)
    g_ref, u_ref, hc_ref, hs_ref = [], [], [], []
    cache = {}
    for i, t in enumerate(sample):
        for j in range(k):
            e = int(r["topk_ids"][t, j])
            if e not in cache:
                cache[e] = omoe.dequantize_expert(oq[e], wl.fmt)
            f = omoe.expert_ffn(a_deq[i:i + 1], cache[e], wl.fmt, inputs.S_H)
            g_ref.append(f["gate"][0]); u_ref.append(f["up"][0])
            hc_ref.append(f["h_codes"][0]); hs_ref.append(f["h_sf"][0])
    err_g = rel_fro(dbg[:, :I], np.array(g_ref))
    err_u = rel_fro(dbg[:, I:], np.array(u_ref))
    assert err_g <= 1e-4 and err_u <= 1e-4, (err_g, err_u)
    differ = (h_codes != np.array(hc_ref)) | (np.repeat(h_sf, v, axis=1) != np.repeat(np.array(hs_ref), v, axis=1))
    assert differ.mean() <= 1e-3, differ.mean()
    err_y = rel_fro(yall[sample], ref["y"])
    assert err_y <= 1e-2, err_y
    print(f"{name}: gate {err_g:.2e} up {err_u:.2e} h-diff {differ.mean():.2e} y {err_y:.2e} "
          f"experts touched {(r['counts'] > 0).sum()} rows {R}")
