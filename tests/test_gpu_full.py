"""GPU parity at the full sizes of the named layers (GPU).

Layers (d_model 4096, expert ffn 2560, 384 experts, top-8): decode NVFP4
(T = 64), decode MXFP8 (T = 256), prefill NVFP4 (T = 8192), prefill NVFP4
with Zipf-skewed routing (T = 16384) and prefill MXFP8 (T = 8192), run with
the same ExpertLayer the benchmark times.  Checked against the oracle:
  * routing of every token: top-k ids, softmax weights, counts, offsets and
    the slot permutation, bit-exact;
  * every valid row of two experts, the most loaded one (many 128-row
    blocks, a ragged last block, many tiles per persistent CTA and many turns
    of the K ring) and the highest-numbered one that receives a slot (the
    end of the tile list): activation codes and scales bit-exact; gate/up
    against the float64 product with relative error <= 1e-4 per expert
    (Frobenius) and per row (the largest row error), so a single bad tile
    cannot hide in a norm; at most 1e-3 of the requantized intermediate's
    (code, block scale) pairs differ; the down rows against the float64
    product of the kernel's own intermediate codes (relative Frobenius
    <= 1e-3: one bf16 rounding);
  * 8 sampled tokens (token 0, token T-1, the token in the most loaded
    expert's last row, 5 seeded others): the weight codes of every expert they
    select, and their bf16 output (relative Frobenius error <= 1e-2);
  * on every token: a finite output.
Bars: the benchmark spec's (bit-exact codes, 1e-4 gate/up, 1e-3 of intermediate
codes, 1e-2 on y).  The per-expert errors are printed (run pytest with -s).
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
from helpers import ACT_TR, kb_padded, rel_fro, sfvec, sf_index_rows, tile_offsets, unpack_codes

FULL = ["decode_nvfp4", "decode_mxfp8", "prefill_nvfp4", "prefill_nvfp4_skewed", "prefill_mxfp8"]
N_SAMPLE = 8


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


def sf_rows(t, rows, nsf):
    """Block scales [len(rows), nsf] of the given rows of a device scale buffer."""
    off = torch.as_tensor(sf_index_rows(rows, nsf).reshape(-1), device=t.device)
    return t.reshape(-1).index_select(0, off).cpu().numpy().reshape(len(rows), nsf)


def sample_tokens(r, T, k, rng):
    """Token 0, token T-1, the token in the most loaded expert's last row and
    seeded others, N_SAMPLE distinct tokens in all (fewer only if T is smaller)."""
    hot = int(np.argmax(r["counts"]))
    last_row = int(r["offsets"][hot]) + int(r["counts"][hot]) - 1
    picks = [0, T - 1, int(r["sorted_slots"][last_row]) // k]
    seen = set(picks)
    for t in rng.permutation(T):
        if len(seen) >= min(N_SAMPLE, T):
            break
        if int(t) not in seen:
            seen.add(int(t))
    return sorted(seen)


def check_expert_rows(layer, wl, r, x_f32, e, q_e):
    """Every valid row of expert e against the oracle; returns the errors."""
    k, H, I, v, fmt = wl.top_k, wl.d_model, wl.d_ffn, sfvec(wl.fmt), wl.fmt
    lo, cnt = int(r["offsets"][e]), int(r["counts"][e])
    rows = np.arange(lo, lo + cnt, dtype=np.int64)
    tokens = r["sorted_slots"][rows] // k
    # activation codes: the oracle's quantization of each row's token
    a_ref, as_ref = omoe.quantize_rows(x_f32[tokens], fmt, inputs.S_X)
    np.testing.assert_array_equal(tiled_rows(layer.a_codes, rows, H, fmt), a_ref, err_msg=f"A codes e={e}")
    np.testing.assert_array_equal(sf_rows(layer.a_sf, rows, H // v), as_ref, err_msg=f"A scales e={e}")
    deq = omoe.dequantize_expert(q_e, fmt)
    f = omoe.expert_ffn(omoe.dequantize_rows(a_ref, as_ref, fmt, inputs.S_X), deq, fmt, inputs.S_H)
    dbg = rows_np(layer.gateup_debug, rows).astype(np.float64)
    gu_ref = np.concatenate([f["gate"], f["up"]], axis=1)
    err = {"rows": cnt, "gate": rel_fro(dbg[:, :I], f["gate"]), "up": rel_fro(dbg[:, I:], f["up"])}
    row_err = np.linalg.norm(dbg - gu_ref, axis=1) / np.maximum(np.linalg.norm(gu_ref, axis=1), 1e-300)
    err["row_max"] = float(row_err.max())
    err["row_argmax"] = int(rows[int(row_err.argmax())])
    # the requantized intermediate
    hc = tiled_rows(layer.h_codes, rows, I, fmt)
    hs = sf_rows(layer.h_sf, rows, I // v)
    differ = (hc != f["h_codes"]) | (np.repeat(hs, v, axis=1) != np.repeat(f["h_sf"], v, axis=1))
    err["h_diff"] = float(differ.mean())
    # down rows: the float64 product of the kernel's own intermediate codes
    o_ref = ofm.bf16_round(omoe.dequantize_rows(hc, hs, fmt, inputs.S_H) @ deq["down"].T)
    o_gpu = layer.down_out.index_select(0, torch.as_tensor(rows, device=layer.down_out.device)).float().cpu().numpy()
    err["down"] = rel_fro(o_gpu, o_ref)
    return err


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
    T, k, E = wl.T, wl.top_k, wl.num_experts

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

    rng = np.random.default_rng(T)
    sample = sample_tokens(r, T, k, rng)
    assert len(sample) == min(N_SAMPLE, T) and 0 in sample and T - 1 in sample
    touched = np.nonzero(r["counts"])[0]
    hot, last = int(np.argmax(r["counts"])), int(touched.max())
    need = sorted(set(int(e) for t in sample for e in r["topk_ids"][t]) | {hot, last})
    oq = oracle_experts(wl, need, dev)
    for e in need:
        assert_expert_equal(gpu_expert(layer, wl, e), oq[e], e)

    # every row of the most loaded and of the last touched expert
    x_f32 = x.float().numpy()
    for e in sorted({hot, last}):
        err = check_expert_rows(layer, wl, r, x_f32, e, oq[e])
        print(f"{name} expert {e}: {err}")
        assert err["gate"] <= 1e-4 and err["up"] <= 1e-4, (e, err)
        assert err["row_max"] <= 1e-4, (e, err)
        assert err["h_diff"] <= 1e-3, (e, err)
        assert err["down"] <= 1e-3, (e, err)

    # the layer output on the sampled tokens
    ref = omoe.forward_tokens(x[sample].float().numpy(), lg[sample].numpy(), oq, k, wl.fmt, inputs.S_X, inputs.S_H)
    err_y = rel_fro(yall[sample], ref["y"])
    print(f"{name}: y {err_y:.2e} on tokens {sample}; experts touched {len(touched)}, rows {R}")
    assert err_y <= 1e-2, err_y
