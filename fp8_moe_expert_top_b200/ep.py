"""Expert parallelism: the routed-expert layer with its experts split over
the ranks of a process group, one GPU per rank.

Page "thinkingmachines/Inkling-2-Small" (vLLM recipe), section Overview, and
page "Thinking Machines releases Inkling 2 Small weights under Apache 2.0",
section "vLLM serving and context limits": the 384 experts are served with
expert parallelism along the tensor-parallel group (EP4, EP8).

Rank g holds experts [g E/G, (g+1) E/G) (E_loc = E/G of them) and routes its
own tokens.  One step on every rank:
  1. route + permute (kernels): the quantized rows of A are grouped by
     expert over all E experts, each expert's segment padded to 128 rows, so
     the rows bound for rank d form one contiguous run of whole 128-row
     blocks, and so do their codes (tiles of 128 rows) and block scales
     (512-byte atoms of 128 rows): both are contiguous byte ranges;
  2. counts: an all-to-all of the per-expert slot counts (E_loc per pair of
     ranks), read back to the host to size the exchanges;
  3. dispatch: an all-to-all(v) of the code bytes and one of the scale bytes
     (quantized rows cross the links, 4x fewer bytes than bf16 for NVFP4);
  4. the grouped expert FFN (moe_forward_grouped): row group (s, e) holds the
     rows rank s sent for local expert e, computed with that expert's weights;
  5. return: an all-to-all(v) of the bf16 output rows back to the rank and
     the rows they came from;
  6. the weighted combine (kernel), unchanged.
Every row is computed exactly as on a single GPU, so each rank's output
equals the single-GPU layer's on its tokens bit for bit.

The exchanges go through torch.distributed (NCCL on GPUs, gloo on CPU);
nothing here loads another GPU's memory directly.  The plan (split sizes,
row groups) is plain host arithmetic on the exchanged counts.
"""

from dataclasses import dataclass

import numpy as np
import torch

from . import binding as B

ROW_ALIGN = 128


def expert_slice(rank, world, num_experts):
    """[first, last) experts held by `rank` of `world` ranks."""
    if num_experts % world:
        raise ValueError(f"{num_experts} experts do not split evenly over {world} ranks")
    n = num_experts // world
    return rank * n, (rank + 1) * n


def _pad(c):
    return (np.asarray(c, dtype=np.int64) + ROW_ALIGN - 1) // ROW_ALIGN * ROW_ALIGN


@dataclass
class DispatchPlan:
    """Sizes of one step's exchanges and the receive-side row groups.

    send_rows[d]   rows (whole 128-row blocks) this rank sends to rank d:
                   its segments of rank d's experts, in expert order
    recv_rows[s]   rows received from rank s, in the same layout
    group_counts   int32 [G * E_loc]: rows in use of group s * E_loc + e
                   (rank s's slots for local expert e)
    group_offsets  int32 [G * E_loc + 1]: first row of each group in the
                   receive buffer (sources in rank order, experts in order)
    group_expert   int32 [G * E_loc]: local expert of each group
    """
    send_rows: list
    recv_rows: list
    group_counts: np.ndarray
    group_offsets: np.ndarray
    group_expert: np.ndarray


def plan_from_counts(counts_to, counts_from):
    """The plan of one step from this rank's per-expert slot counts
    counts_to [G, E_loc] (row d: the experts of rank d) and the counts the
    other ranks send for this rank's experts, counts_from [G, E_loc]."""
    counts_to = np.asarray(counts_to, dtype=np.int64)
    counts_from = np.asarray(counts_from, dtype=np.int64)
    if counts_to.shape != counts_from.shape or counts_to.ndim != 2:
        raise ValueError(f"count tables {counts_to.shape} / {counts_from.shape}")
    G, E_loc = counts_from.shape
    send_rows = [int(v) for v in _pad(counts_to).sum(axis=1)]
    recv_rows = [int(v) for v in _pad(counts_from).sum(axis=1)]
    group_counts = counts_from.reshape(-1)
    group_offsets = np.concatenate([[0], np.cumsum(_pad(group_counts))])
    group_expert = np.tile(np.arange(E_loc, dtype=np.int64), G)
    return DispatchPlan(send_rows, recv_rows, group_counts.astype(np.int32), group_offsets.astype(np.int32),
                        group_expert.astype(np.int32))


def exchange_counts(counts, world, group=None):
    """counts [E] int32 (this rank's slots per expert, all experts) ->
    counts_from [G, E_loc] numpy: row s = the counts rank s has for this
    rank's experts.  Synchronizes with the host (the split sizes of the row
    exchanges must be known there)."""
    import torch.distributed as dist
    out = torch.empty_like(counts)
    if world == 1:
        out.copy_(counts)
    else:
        dist.all_to_all_single(out, counts, group=group)
    return out.cpu().numpy().reshape(world, -1)


def exchange_rows(recv, send, recv_rows, send_rows, row_bytes, group=None):
    """All-to-all(v) of whole rows between flat byte tensors: send[sum of
    send_rows rows] goes out, send_rows[d] rows to rank d, and recv gets
    recv_rows[s] rows from rank s, in rank order; a row is row_bytes bytes."""
    import torch.distributed as dist
    n_out, n_in = sum(recv_rows) * row_bytes, sum(send_rows) * row_bytes
    if len(send_rows) == 1:
        recv[:n_out].copy_(send[:n_in])
        return
    dist.all_to_all_single(recv[:n_out], send[:n_in], output_split_sizes=[r * row_bytes for r in recv_rows],
                           input_split_sizes=[r * row_bytes for r in send_rows], group=group)


def _bytes(t):
    return t.reshape(-1).view(torch.uint8)


class ExpertParallelLayer:
    """One rank's part of the expert-parallel layer (GPU).

    Buffers for up to T_max local tokens (and for the rows of up to
    T_peer_max tokens from each rank); routing over all num_experts; packed
    weights of this rank's num_experts / G experts only.  forward()
    runs the six steps above on the current stream; the phases are also
    exposed (local_begin, plan, experts, local_end) with the exchanges left to
    the caller, for callers that move the bytes themselves.
    """

    def __init__(self, num_experts, top_k, d_model, d_ffn, fmt, T_max, device, rank=0, world=1, group=None,
                 s_x=None, s_h=None, T_peer_max=None):
        self.E, self.k, self.H, self.I = num_experts, top_k, d_model, d_ffn
        self.rank, self.G, self.group = rank, world, group
        self.e0, self.e1 = expert_slice(rank, world, num_experts)
        self.E_loc = self.e1 - self.e0
        self.cfg = B.make_config(num_experts, top_k, d_model, d_ffn, fmt)
        # this rank's experts; a token reaches at most min(k, E_loc) of them
        self.cfg_loc = B.make_config(self.E_loc, min(top_k, self.E_loc), d_model, d_ffn, fmt)
        for c in (self.cfg, self.cfg_loc):
            st = B.moe_check_config(c)
            if st != 0:
                raise B.MoeError("moe_check_config", st, B.lib().moe_status_string(st).decode())
        self.fmt = self.cfg.fmt
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError(f"ExpertParallelLayer runs on a CUDA device, not {self.device}")
        dev = self.device
        self.T_max = int(T_max)
        T, k, E, H, I = self.T_max, top_k, num_experts, d_model, d_ffn
        self.layout = B.moe_get_weights_layout(self.cfg_loc)
        self.packed = torch.empty(self.layout.total_bytes, dtype=torch.uint8, device=dev)
        # routing and the send side, over all experts
        self.R_max = B.moe_max_rows(self.cfg, T)
        i32 = dict(dtype=torch.int32, device=dev)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.topk_ids = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.sorted_slots = torch.empty(self.R_max, **i32)
        self.slot_to_row = torch.empty(T * k, **i32)
        self.route_ws = torch.empty(B.moe_route_workspace_bytes(self.cfg, T), **u8)
        self.a_codes = torch.empty(B.moe_codes_bytes(self.cfg, self.R_max, H), **u8)
        self.a_sf = torch.empty(B.moe_sf_bytes(self.cfg, self.R_max, H), **u8)
        self.o_local = torch.empty(self.R_max, H, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        # the receive side: every rank may send all its slots here (up to
        # T_peer_max tokens per rank, T_max by default)
        per_src = B.moe_max_rows(self.cfg_loc, T if T_peer_max is None else int(T_peer_max))
        self.R_recv = world * per_src
        self.r_codes = torch.empty(B.moe_codes_bytes(self.cfg, self.R_recv, H), **u8)
        self.r_sf = torch.empty(B.moe_sf_bytes(self.cfg, self.R_recv, H), **u8)
        self.h_codes = torch.empty(B.moe_codes_bytes(self.cfg, self.R_recv, I), **u8)
        self.h_sf = torch.empty(B.moe_sf_bytes(self.cfg, self.R_recv, I), **u8)
        self.o_recv = torch.empty(self.R_recv, H, dtype=torch.bfloat16, device=dev)
        n_groups = world * self.E_loc
        self.group_offsets = torch.zeros(n_groups + 1, **i32)
        self.group_counts = torch.zeros(n_groups, **i32)
        self.group_expert = torch.zeros(n_groups, **i32)
        self.status = torch.zeros(1, **i32)
        f32 = dict(dtype=torch.float32, device=dev)
        if self.fmt == B.MOE_NVFP4:
            if s_x is None or s_h is None:
                raise ValueError("NVFP4 needs the static activation scales s_x and s_h")
            self.act_scale = torch.tensor([float(s_x)], **f32)
            self.inter_scale = torch.tensor([float(s_h)], **f32)
        else:
            self.act_scale = self.inter_scale = None
        self.kb_h = B.moe_codes_bytes(self.cfg, ROW_ALIGN, H) // ROW_ALIGN   # code bytes per row of A
        self.sf_h = B.moe_sf_bytes(self.cfg, ROW_ALIGN, H) // ROW_ALIGN      # scale bytes per row of A
        self.plan_ = None

    # ------------------------------------------------------------- weights
    def quantize_experts(self, local_begin, w_gate, w_up, w_down):
        """Quantize float32 weights of local experts [local_begin, local_begin
        + n) (global experts e0 + local_begin ...) into this rank's slice."""
        n = w_gate.shape[0]
        if local_begin < 0 or local_begin + n > self.E_loc:
            raise ValueError(f"local experts {local_begin}..{local_begin + n} outside 0..{self.E_loc}")
        B.moe_quantize_weights(self.cfg_loc, local_begin, n, w_gate, w_up, w_down, self.packed)

    # ------------------------------------------------------------- phases
    def local_begin(self, x, logits, T):
        """Route this rank's T tokens over all experts and quantize their rows."""
        if not 0 <= T <= self.T_max:
            raise ValueError(f"T = {T} tokens, buffers hold 0..{self.T_max}")
        self.T = T
        B.moe_route_topk(self.cfg, T, logits, self.topk_ids, self.topk_w, self.expert_counts, self.expert_offsets,
                         self.sorted_slots, self.slot_to_row, self.route_ws)
        B.moe_permute(self.cfg, T, x, self.act_scale, self.slot_to_row, self.a_codes, self.a_sf)

    def counts_to(self):
        """[G, E_loc] numpy: this rank's slot counts, by destination rank (host sync)."""
        return self.expert_counts.cpu().numpy().reshape(self.G, self.E_loc)

    def plan(self, counts_from):
        """Size the exchanges and set the row groups from the counts the
        ranks send for this rank's experts ([G, E_loc])."""
        p = plan_from_counts(self.counts_to(), counts_from)
        if sum(p.recv_rows) > self.R_recv:
            raise ValueError(f"{sum(p.recv_rows)} received rows exceed the buffers' {self.R_recv}")
        self.group_offsets.copy_(torch.from_numpy(p.group_offsets))
        self.group_counts.copy_(torch.from_numpy(p.group_counts))
        self.group_expert.copy_(torch.from_numpy(p.group_expert))
        self.plan_ = p
        return p

    def experts(self):
        """The grouped expert FFN over the received rows."""
        B.moe_forward_grouped(self.cfg_loc, self.G * self.E_loc, self.R_recv, self.packed, self.r_codes, self.r_sf,
                              self.act_scale, self.inter_scale, self.group_offsets, self.group_counts,
                              self.group_expert, self.h_codes, self.h_sf, self.o_recv, None, self.status)

    def local_end(self):
        """The weighted combine of this rank's tokens from their returned rows."""
        B.moe_unpermute_combine(self.cfg, self.T, self.o_local, self.topk_w, self.slot_to_row, self.y)
        return self.y[:self.T]

    # byte views of the exchanged buffers
    def send_views(self):
        return _bytes(self.a_codes), _bytes(self.a_sf)

    def recv_views(self):
        return _bytes(self.r_codes), _bytes(self.r_sf)

    # ------------------------------------------------------------- one step
    def forward(self, x, logits):
        """y [T, H] of this rank's tokens x [T, H] bf16, logits [T, E] fp32."""
        T = x.shape[0]
        self.local_begin(x, logits, T)
        p = self.plan(exchange_counts(self.expert_counts, self.G, self.group))
        sc, ss = self.send_views()
        rc, rs = self.recv_views()
        exchange_rows(rc, sc, p.recv_rows, p.send_rows, self.kb_h, self.group)
        exchange_rows(rs, ss, p.recv_rows, p.send_rows, self.sf_h, self.group)
        self.experts()
        row = 2 * self.H
        exchange_rows(_bytes(self.o_local), _bytes(self.o_recv), p.send_rows, p.recv_rows, row, self.group)
        return self.local_end()
