"""Expert-parallel plumbing on CPU (gloo, two and four ranks).

The exchanges of fp8_moe_expert_top_b200.ep (counts, dispatch of the
quantized rows as whole 128-row blocks of tiled codes and scale atoms,
return of the output rows) and its plan (split sizes, row groups) are the
host side of the expert-parallel layer.  Here gloo ranks (two, and four with
uneven token counts) run them on CPU
tensors laid out exactly as the kernels lay them out, with the oracle
standing in for the kernels on each rank (routing, quantized rows, each
received group's expert FFN, the combine).  Checked:
  * every received row group (s, e) holds, bit for bit, the codes and block
    scales of rank s's tokens routed to local expert e, in token order;
  * each rank's output equals the oracle's single-process forward over the
    tokens of all ranks, on that rank's tokens;
  * the plan alone, on random and edge-case counts (empty experts, a rank
    that sends nothing).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from fp8_moe_expert_top_b200 import ep, inputs
from oracle import moe as omoe
from oracle import route as ort

from helpers import ACT_TR, kb_padded, pack_nvfp4, pad_row_bytes, sfvec, swizzle_sf, tile_matrix, tiled_codes, \
    unswizzle_sf

WL = inputs.WORKLOADS["tiny_nvfp4"]
TOKENS = (40, 57, 3, 13)   # tokens of ranks 0..3 (the first `world` are used)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(rank, fmt):
    T = TOKENS[rank]
    x = inputs.make_x(WL, seed=inputs.BASE_SEED + 10 + rank, T=T).float().numpy()
    lg = inputs.make_logits(WL, seed=inputs.BASE_SEED + 20 + rank, T=T).numpy()
    return x, lg


def _experts(fmt):
    return {e: omoe.quantize_expert(*(w.numpy() for w in inputs.make_expert_weights(WL, e)), fmt)
            for e in range(WL.num_experts)}


def _send_buffers(x, lg, fmt):
    """Routing of one rank's tokens and its rows of A in the kernels' byte layout."""
    k, E, H = WL.top_k, WL.num_experts, WL.d_model
    r = ort.route(lg, k, E)
    codes, sf = omoe.quantize_rows(x, fmt, inputs.S_X)
    R = int(r["offsets"][-1])
    rows_c = np.zeros((R, H), dtype=np.uint8)
    rows_s = np.zeros((R, H // sfvec(fmt)), dtype=np.uint8)
    valid = r["sorted_slots"] >= 0
    tok = r["sorted_slots"][valid] // k
    rows_c[valid], rows_s[valid] = codes[tok], sf[tok]
    raw = pack_nvfp4(rows_c) if fmt == "nvfp4" else rows_c
    a_codes = tile_matrix(pad_row_bytes(raw, kb_padded(H, fmt)), ACT_TR)
    a_sf = swizzle_sf(rows_s)
    return r, codes, sf, torch.from_numpy(a_codes), torch.from_numpy(a_sf)


def _rank_main(rank, world, port, fmt, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        k, E, H = WL.top_k, WL.num_experts, WL.d_model
        v, kb = sfvec(fmt), kb_padded(H, fmt)
        e0, e1 = ep.expert_slice(rank, world, E)
        E_loc = e1 - e0
        experts = _experts(fmt)
        x, lg = _rank_inputs(rank, fmt)
        r, _, _, a_codes, a_sf = _send_buffers(x, lg, fmt)
        counts_from = ep.exchange_counts(torch.from_numpy(r["counts"].astype(np.int32)), world)
        plan = ep.plan_from_counts(r["counts"].reshape(world, E_loc), counts_from)
        R_recv = int(plan.group_offsets[-1])
        r_codes = torch.zeros(R_recv * kb, dtype=torch.uint8)
        r_sf = torch.zeros(R_recv * (H // v), dtype=torch.uint8)
        ep.exchange_rows(r_codes, a_codes, plan.recv_rows, plan.send_rows, kb)
        ep.exchange_rows(r_sf, a_sf, plan.recv_rows, plan.send_rows, H // v)
        got_c = tiled_codes(fmt, r_codes.numpy(), np.arange(R_recv), H, ACT_TR)
        got_s = unswizzle_sf(r_sf.numpy(), R_recv, H // v)
        # each group: rank s's tokens of local expert e, in token order
        o_recv = np.zeros((R_recv, H), dtype=np.float64)
        for s in range(world):
            xs, lgs = _rank_inputs(s, fmt)
            rs = ort.route(lgs, k, E)
            cs, ss = omoe.quantize_rows(xs, fmt, inputs.S_X)
            for e in range(E_loc):
                g = s * E_loc + e
                off, cnt = int(plan.group_offsets[g]), int(plan.group_counts[g])
                assert int(plan.group_expert[g]) == e
                toks = np.nonzero((rs["topk_ids"] == e0 + e).any(axis=1))[0]
                assert cnt == len(toks)
                np.testing.assert_array_equal(got_c[off:off + cnt], cs[toks])
                np.testing.assert_array_equal(got_s[off:off + cnt], ss[toks])
                if cnt:
                    a_deq = omoe.dequantize_rows(got_c[off:off + cnt], got_s[off:off + cnt], fmt, inputs.S_X)
                    f = omoe.expert_ffn(a_deq, omoe.dequantize_expert(experts[e0 + e], fmt), fmt, inputs.S_H)
                    o_recv[off:off + cnt] = f["out"]
        R = int(r["offsets"][-1])
        o_local = torch.full((R, H), np.nan, dtype=torch.float64)
        ep.exchange_rows(o_local.view(-1).view(torch.uint8), torch.from_numpy(o_recv).view(-1).view(torch.uint8),
                         plan.send_rows, plan.recv_rows, H * 8)
        y = omoe.combine(o_local.numpy(), r["topk_w"], r["slot_to_row"])
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fmt,world", [("nvfp4", 2), ("mxfp8", 2), ("nvfp4", 4)])
def test_ep_ranks_match_single_process(tmp_path, fmt, world):
    for _ in range(3):            # the probed port can be taken before gloo binds it
        try:
            mp.start_processes(_rank_main, args=(world, _free_port(), fmt, str(tmp_path)), nprocs=world,
                               start_method="spawn")
            break
        except Exception as exc:  # noqa: BLE001
            if "address" not in str(exc).lower():
                raise
    xs, lgs = zip(*(_rank_inputs(r, fmt) for r in range(world)))
    ref = omoe.forward(np.concatenate(xs), np.concatenate(lgs), _experts(fmt), WL.top_k, fmt, inputs.S_X,
                       inputs.S_H, WL.num_experts)["y"]
    t0 = 0
    for rank in range(world):
        y = np.load(tmp_path / f"y{rank}.npy")
        yr = ref[t0:t0 + TOKENS[rank]]
        t0 += TOKENS[rank]
        assert y.shape == yr.shape
        assert np.linalg.norm(y - yr) <= 1e-6 * np.linalg.norm(yr)


def test_plan_from_counts():
    rng = np.random.default_rng(5)
    for G, E_loc in ((1, 8), (2, 4), (4, 96), (8, 48)):
        to = rng.integers(0, 300, (G, E_loc))
        fr = rng.integers(0, 300, (G, E_loc))
        to[0] = 0                                  # a rank that sends nothing to rank 0
        fr[:, -1] = 0                              # an expert nobody routes to
        p = ep.plan_from_counts(to, fr)
        pad = lambda c: (c + 127) // 128 * 128     # noqa: E731
        assert p.send_rows == [int(pad(to[d]).sum()) for d in range(G)]
        assert p.recv_rows == [int(pad(fr[s]).sum()) for s in range(G)]
        assert p.group_offsets[0] == 0 and np.all(np.diff(p.group_offsets) % 128 == 0)
        np.testing.assert_array_equal(np.diff(p.group_offsets), pad(fr.reshape(-1)))
        np.testing.assert_array_equal(p.group_counts, fr.reshape(-1))
        np.testing.assert_array_equal(p.group_expert, np.tile(np.arange(E_loc), G))
        # the groups of source s fill exactly its received rows
        ends = np.cumsum(p.recv_rows)
        np.testing.assert_array_equal(p.group_offsets[E_loc::E_loc], ends)
    with pytest.raises(ValueError):
        ep.plan_from_counts(np.zeros((2, 4)), np.zeros((4, 2)))
    with pytest.raises(ValueError):
        ep.expert_slice(0, 5, 384)
