"""Expert-parallel layer on one GPU (GPU).

G ranks of fp8_moe_expert_top_b200.ep.ExpertParallelLayer are emulated in
one process on one GPU: each holds E/G experts and its own tokens, and the
exchanges between them are done here as plain device copies following each
rank's plan (what the all-to-alls move between GPUs).  No kernel of one
emulated rank waits on another's.  This runs the kernel side of expert
parallelism (routing over all experts, the rows of each destination as whole
128-row blocks, the grouped FFN over rows grouped by (source rank, local
expert), the return of the output rows, the combine) and checks each rank's
output against the single-GPU layer on the same tokens: every row is
computed the same way, so they must be equal bit for bit.  A one-rank layer
runs its own forward() (no process group needed for one rank).
"""

import dataclasses

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from fp8_moe_expert_top_b200 import ep, inputs

from gpu_common import build_layer


def _ranks(wl, G, tokens, dev):
    ranks = []
    for g in range(G):
        r = ep.ExpertParallelLayer(wl.num_experts, wl.top_k, wl.d_model, wl.d_ffn, wl.fmt, tokens[g], dev, rank=g,
                                   world=G, s_x=inputs.S_X, s_h=inputs.S_H, T_peer_max=max(tokens))
        chunk = 16
        for l0 in range(0, r.E_loc, chunk):
            n = min(chunk, r.E_loc - l0)
            ws = [inputs.make_expert_weights(wl, r.e0 + l0 + i, device=dev) for i in range(n)]
            r.quantize_experts(l0, *(torch.stack([w[m] for w in ws]).contiguous() for m in range(3)))
            del ws
        ranks.append(r)
    torch.cuda.synchronize()
    return ranks


def _exchange(ranks, send, recv, row_bytes, back=False):
    """Emulated all-to-all(v) of whole rows between the ranks' byte buffers."""
    G = len(ranks)
    for d in range(G):
        pos = 0
        for s in range(G):
            ps = ranks[s].plan_
            if not back:   # rows rank s sends to d: its segment of d's experts
                n, start = ps.send_rows[d], sum(ps.send_rows[:d])
            else:          # rows rank s returns to d: the rows it received from d
                n, start = ps.recv_rows[d], sum(ps.recv_rows[:d])
            recv(d)[pos * row_bytes:(pos + n) * row_bytes].copy_(send(s)[start * row_bytes:(start + n) * row_bytes])
            pos += n
        pd = ranks[d].plan_
        assert pos == (sum(pd.recv_rows) if not back else sum(pd.send_rows))


def _emulated_forward(ranks, xs, lgs):
    G, E_loc = len(ranks), ranks[0].E_loc
    for r, x, lg in zip(ranks, xs, lgs):
        r.local_begin(x, lg, x.shape[0])
    counts = [r.expert_counts.cpu().numpy() for r in ranks]
    for g, r in enumerate(ranks):
        r.plan(np.stack([counts[s][g * E_loc:(g + 1) * E_loc] for s in range(G)]))
    _exchange(ranks, lambda s: ranks[s].send_views()[0], lambda d: ranks[d].recv_views()[0], ranks[0].kb_h)
    _exchange(ranks, lambda s: ranks[s].send_views()[1], lambda d: ranks[d].recv_views()[1], ranks[0].sf_h)
    for r in ranks:
        r.experts()
    _exchange(ranks, lambda s: ranks[s].o_recv.view(-1).view(torch.uint8),
              lambda d: ranks[d].o_local.view(-1).view(torch.uint8), 2 * ranks[0].H, back=True)
    return [r.local_end() for r in ranks]


CASES = [("tiny_nvfp4", 2, (40, 57)), ("tiny_nvfp4", 4, (1, 30, 0, 64)), ("decode_nvfp4", 2, (64, 100)),
         ("decode_mxfp8", 4, (256, 64, 128, 32))]


@pytest.mark.gpu
@pytest.mark.parametrize("name,G,tokens", CASES)
def test_ep_emulated_ranks_match_single_gpu(cuda_device, name, G, tokens):
    dev = cuda_device
    wl = inputs.WORKLOADS[name]
    T = sum(tokens)
    ref = build_layer(dataclasses.replace(wl, T=T), dev, debug=False, weight_device=dev)
    x = inputs.make_x(wl, seed=inputs.BASE_SEED + 77, T=T).to(dev)
    lg = inputs.make_logits(wl, seed=inputs.BASE_SEED + 78, T=T).to(dev)
    y_ref = ref.forward(x, lg).clone()
    torch.cuda.synchronize()
    assert int(ref.status.item()) == 0
    del ref
    torch.cuda.empty_cache()
    ranks = _ranks(wl, G, tokens, dev)
    bounds = np.concatenate([[0], np.cumsum(tokens)])
    xs = [x[bounds[g]:bounds[g + 1]].contiguous() for g in range(G)]
    lgs = [lg[bounds[g]:bounds[g + 1]].contiguous() for g in range(G)]
    ys = _emulated_forward(ranks, xs, lgs)
    torch.cuda.synchronize()
    for g, (r, y) in enumerate(zip(ranks, ys)):
        assert int(r.status.item()) == 0, g
        assert torch.equal(y, y_ref[bounds[g]:bounds[g + 1]]), g
    # a second step with other tokens reuses the buffers and plans afresh
    x2 = inputs.make_x(wl, seed=inputs.BASE_SEED + 79, T=T).to(dev)
    lg2 = inputs.make_logits(wl, seed=inputs.BASE_SEED + 80, T=T).to(dev)
    ys2 = _emulated_forward(ranks, [x2[bounds[g]:bounds[g + 1]].contiguous() for g in range(G)],
                            [lg2[bounds[g]:bounds[g + 1]].contiguous() for g in range(G)])
    del ranks
    torch.cuda.empty_cache()
    ref = build_layer(dataclasses.replace(wl, T=T), dev, debug=False, weight_device=dev)
    y2_ref = ref.forward(x2, lg2)
    torch.cuda.synchronize()
    for g, y in enumerate(ys2):
        assert torch.equal(y, y2_ref[bounds[g]:bounds[g + 1]]), g


@pytest.mark.gpu
def test_ep_single_rank_forward(cuda_device):
    dev = cuda_device
    wl = inputs.WORKLOADS["tiny_nvfp4"]
    ref = build_layer(wl, dev, debug=False, weight_device=dev)   # the ranks draw their weights on the device too
    x, lg = inputs.make_x(wl).to(dev), inputs.make_logits(wl).to(dev)
    y_ref = ref.forward(x, lg).clone()
    (r,) = _ranks(wl, 1, (wl.T,), dev)
    y = r.forward(x, lg)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)


@pytest.mark.gpu
def test_grouped_forward_reports_an_expert_outside_the_weights(cuda_device):
    """A group naming an expert the packed weights do not hold is computed
    with expert 0's weights (no out-of-range read) and flagged."""
    dev = cuda_device
    wl = inputs.WORKLOADS["tiny_nvfp4"]
    (r,) = _ranks(wl, 1, (wl.T,), dev)
    x, lg = inputs.make_x(wl).to(dev), inputs.make_logits(wl).to(dev)
    r.forward(x, lg)
    torch.cuda.synchronize()
    r.group_expert.fill_(wl.num_experts + 5)
    r.status.zero_()
    r.experts()
    torch.cuda.synchronize()
    assert int(r.status.item()) & B.MOE_DEVICE_BAD_GROUP_EXPERT
