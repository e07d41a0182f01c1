"""ExpertLayer: device buffers plus the four calls of one routed-expert layer.

This is the public Python entry point a user calls: it owns PyTorch-allocated
device buffers sized for up to T_max tokens and runs, on the current stream,

    moe_route_topk -> moe_permute -> moe_forward -> moe_unpermute_combine

through the C ABI.  Nothing here computes any part of the layer.
"""

import torch

from . import binding as B


class ExpertLayer:
    def __init__(self, num_experts, top_k, d_model, d_ffn, fmt, T_max, device, s_x=None, s_h=None,
                 debug=False):
        self.cfg = B.make_config(num_experts, top_k, d_model, d_ffn, fmt)
        st = B.moe_check_config(self.cfg)
        if st != 0:
            raise B.MoeError("moe_check_config", st, B.lib().moe_status_string(st).decode())
        self.E, self.k, self.H, self.I = num_experts, top_k, d_model, d_ffn
        self.fmt = self.cfg.fmt
        self.T_max = int(T_max)
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError(f"ExpertLayer runs on a CUDA device, not {self.device}")
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        if self.T_max < 0:
            raise ValueError(f"T_max must be >= 0, got {self.T_max}")
        dev = self.device
        self.layout = B.moe_get_weights_layout(self.cfg)
        self.packed = torch.empty(self.layout.total_bytes, dtype=torch.uint8, device=dev)
        self.R_max = B.moe_max_rows(self.cfg, self.T_max)
        R, T, k, E, H, I = self.R_max, self.T_max, top_k, num_experts, d_model, d_ffn
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_ids = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.sorted_slots = torch.empty(R, **i32)
        self.slot_to_row = torch.empty(T * k, **i32)
        self.route_ws = torch.empty(B.moe_route_workspace_bytes(self.cfg, T), dtype=torch.uint8, device=dev)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.a_codes = torch.empty(B.moe_codes_bytes(self.cfg, R, H), **u8)
        self.h_codes = torch.empty(B.moe_codes_bytes(self.cfg, R, I), **u8)
        if self.cfg.fmt == B.MOE_BF16:   # no block scales
            self.a_sf = self.h_sf = None
        else:
            self.a_sf = torch.empty(B.moe_sf_bytes(self.cfg, R, H), **u8)
            self.h_sf = torch.empty(B.moe_sf_bytes(self.cfg, R, I), **u8)
        self.down_out = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, **i32)
        self.gateup_debug = torch.empty(R, 2 * I, dtype=torch.float32, device=dev) if debug else None
        f32 = dict(dtype=torch.float32, device=dev)
        if self.fmt == B.MOE_BF16:
            self.act_scale = None
            self.inter_scale = None
        elif self.fmt == B.MOE_NVFP4:
            if s_x is None or s_h is None:
                raise ValueError("NVFP4 needs the static activation scales s_x and s_h")
            self.act_scale = torch.tensor([float(s_x)], **f32)
            self.inter_scale = torch.tensor([float(s_h)], **f32)
        else:
            self.act_scale = None
            self.inter_scale = None

    # ------------------------------------------------------------- weights
    def quantize_experts(self, expert_begin, w_gate, w_up, w_down):
        """Quantize float32 weights of experts [begin, begin + n) into self.packed."""
        n = w_gate.shape[0]
        shapes = ((n, self.I, self.H), (n, self.I, self.H), (n, self.H, self.I))
        for name, t, shape in zip(("w_gate", "w_up", "w_down"), (w_gate, w_up, w_down), shapes):
            if t.dtype != torch.float32 or tuple(t.shape) != shape:
                raise ValueError(f"{name}: float32 {shape} expected, got {t.dtype} {tuple(t.shape)}")
        B.moe_quantize_weights(self.cfg, expert_begin, n, w_gate, w_up, w_down, self.packed)

    def pack_experts_bf16(self, expert_begin, w_gate, w_up, w_down, lora=None, lora_rank=0, lora_scaling=0.0):
        """BF16 layers: bf16 weights of experts [begin, begin + n) and their
        adapters lora = (A_gate, B_gate, A_up, B_up, A_down, B_down) (bf16,
        [n, r, H], [n, I, r], [n, r, H], [n, I, r], [n, r, I], [n, H, r]) or
        None, into self.packed."""
        if self.fmt != B.MOE_BF16:
            raise ValueError("pack_experts_bf16 is for BF16 layers (quantize_experts for NVFP4 / MXFP8)")
        n = w_gate.shape[0]
        shapes = [(n, self.I, self.H), (n, self.I, self.H), (n, self.H, self.I)]
        ts = [w_gate, w_up, w_down]
        if lora is not None:
            r = int(lora_rank)
            shapes += [(n, r, self.H), (n, self.I, r), (n, r, self.H), (n, self.I, r), (n, r, self.I), (n, self.H, r)]
            ts += list(lora)
        for i, (t, shape) in enumerate(zip(ts, shapes)):
            if t.dtype != torch.bfloat16 or tuple(t.shape) != shape:
                raise ValueError(f"argument {i}: bfloat16 {shape} expected, got {t.dtype} {tuple(t.shape)}")
        B.moe_pack_weights_bf16(self.cfg, expert_begin, n, w_gate, w_up, w_down, lora, lora_rank, lora_scaling,
                                self.packed)

    # ------------------------------------------------------------- steps
    def _check_T(self, T):
        if not 0 <= T <= self.T_max:
            raise ValueError(f"T = {T} tokens, this layer's buffers hold 0..{self.T_max}")

    def _check_io(self, T, x=None, logits=None, y=None):
        """Shapes, dtypes and device of step inputs / outputs holding >= T rows."""
        self._check_T(T)
        args = [(name, t, cols, dtype) for name, t, cols, dtype in (
            ("x", x, self.H, torch.bfloat16), ("logits", logits, self.E, torch.float32),
            ("y", y, self.H, torch.bfloat16)) if t is not None]
        for name, t, cols, dtype in args:
            if t.dim() != 2 or t.shape[0] < T or t.shape[1] != cols or t.dtype != dtype:
                raise ValueError(f"{name}: {dtype} [>= {T}, {cols}] expected, got {t.dtype} {tuple(t.shape)}")
        for name, t, _, _ in args:
            if t.device != self.device:
                raise ValueError(f"{name} is on {t.device}, the layer on {self.device}")

    def route(self, logits, T):
        B.moe_route_topk(self.cfg, T, logits, self.topk_ids, self.topk_w, self.expert_counts,
                         self.expert_offsets, self.sorted_slots, self.slot_to_row, self.route_ws)

    def set_router(self, w_router):
        """bf16 router weights [E, H] (device) for routing from x (route_x)."""
        if w_router.dtype != torch.bfloat16 or tuple(w_router.shape) != (self.E, self.H):
            raise ValueError(f"w_router: bfloat16 ({self.E}, {self.H}) expected, got {w_router.dtype} "
                             f"{tuple(w_router.shape)}")
        if w_router.device != self.device:
            raise ValueError(f"w_router is on {w_router.device}, the layer on {self.device}")
        self.w_router = w_router.contiguous()

    def route_x(self, x, T, logits_out=None):
        """Routing from the layer input x [>= T, H] bf16: router scores fused
        with the top-k (moe_router_topk)."""
        B.moe_router_topk(self.cfg, T, x, self.w_router, logits_out, self.topk_ids, self.topk_w, self.expert_counts,
                          self.expert_offsets, self.sorted_slots, self.slot_to_row, self.route_ws, self.status)

    def permute(self, x, T):
        B.moe_permute(self.cfg, T, x, self.act_scale, self.slot_to_row, self.a_codes, self.a_sf)

    def experts(self, T):
        B.moe_forward(self.cfg, T, self.packed, self.a_codes, self.a_sf, self.act_scale, self.inter_scale,
                      self.expert_offsets, self.expert_counts, self.h_codes, self.h_sf, self.down_out,
                      self.gateup_debug, self.status)

    def gateup(self, T):
        B.moe_forward_gateup(self.cfg, T, self.packed, self.a_codes, self.a_sf, self.act_scale, self.inter_scale,
                             self.expert_offsets, self.expert_counts, self.h_codes, self.h_sf, self.gateup_debug,
                             self.status)

    def down(self, T):
        B.moe_forward_down(self.cfg, T, self.packed, self.h_codes, self.h_sf, self.inter_scale,
                           self.expert_offsets, self.expert_counts, self.down_out, self.status)

    def combine(self, T, y=None):
        B.moe_unpermute_combine(self.cfg, T, self.down_out, self.topk_w, self.slot_to_row,
                                self.y if y is None else y)

    # ------------------------------------------------------------- graphs
    def capture(self, T, events=None, x_in=None, logits_in=None, y_out=None):
        """Capture the whole layer for T tokens as a CUDA graph.

        The graph reads its inputs from x_in [>= T, H] (bf16) and logits_in
        [>= T, E] (float32) and writes y_out [>= T, H] (bf16); by default
        self.x_in, self.logits_in (allocated here) and self.y.  `events`, if
        given, is a list of six timing events created with external=True; they
        are recorded before the layer and after each of its five steps.  Run
        one eager forward first so that every kernel is set up.
        """
        if getattr(self, "x_in", None) is None:
            self.x_in = torch.zeros(self.T_max, self.H, dtype=torch.bfloat16, device=self.device)
            self.logits_in = torch.zeros(self.T_max, self.E, dtype=torch.float32, device=self.device)
        x_in = self.x_in if x_in is None else x_in
        logits_in = self.logits_in if logits_in is None else logits_in
        y_out = self.y if y_out is None else y_out
        self._check_io(T, x_in, logits_in, y_out)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        steps = (lambda: self.route(logits_in, T), lambda: self.permute(x_in, T),
                 lambda: self.gateup(T), lambda: self.down(T), lambda: self.combine(T, y_out))
        with torch.cuda.graph(g, stream=side):
            if events is not None:
                events[0].record()
            for i, fn in enumerate(steps):
                fn()
                if events is not None:
                    events[i + 1].record()
        torch.cuda.current_stream(self.device).wait_stream(side)
        g.moe_layer_io = (self, T, x_in, logits_in, y_out)
        return g

    def forward_graph(self, graph, x, logits):
        """Copy x [T, H] / logits [T, E] into the input buffers `graph` was
        captured with (by this layer's capture), replay it, and return its
        output rows y[:T]."""
        io = getattr(graph, "moe_layer_io", None)
        if io is None or io[0] is not self:
            raise ValueError("the graph was not captured by this layer's capture()")
        _, T, x_in, logits_in, y_out = io
        if x.shape[0] != T or logits.shape[0] != T:
            raise ValueError(f"the graph was captured for T = {T}, got {x.shape[0]} / {logits.shape[0]} rows")
        self._check_io(T, x, logits)
        x_in[:T].copy_(x, non_blocking=True)
        logits_in[:T].copy_(logits, non_blocking=True)
        graph.replay()
        return y_out[:T]

    def forward(self, x, logits=None):
        """y[:T] for bf16 x [T, H] and float32 logits [T, E] already on the
        device; with logits None the router weights given to set_router score
        the tokens (moe_router_topk)."""
        T = x.shape[0]
        self._check_io(T, x, logits)
        if logits is None:
            if getattr(self, "w_router", None) is None:
                raise ValueError("no logits and no router weights (set_router)")
            self.route_x(x, T)
        else:
            if logits.shape[0] != T:
                raise ValueError(f"x has {T} rows, logits {logits.shape[0]}")
            self.route(logits, T)
        self.permute(x, T)
        self.gateup(T)
        self.down(T)
        self.combine(T)
        return self.y[:T]


class HostPipeline:
    """The layer over a sequence of host batches of T tokens each, with the
    host <-> device copies of neighbouring batches overlapping its kernels.

    Two CUDA graphs of the layer alternate, each with its own device input and
    output buffers.  Batch i's x and logits go up on an upload stream while
    batch i - 1 computes, and each batch's y comes down on a download stream
    while the next one computes.  Events order every reuse of a buffer: a
    slot's inputs are overwritten only after the graph that read them has
    finished, and its output only after it has been copied out.  The graphs
    share the layer's intermediate buffers, so they run one after the other on
    the current stream.
    """

    def __init__(self, layer, T):
        self.layer, self.T = layer, T
        dev = layer.device
        self.x = [torch.zeros(T, layer.H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.logits = [torch.zeros(T, layer.E, dtype=torch.float32, device=dev) for _ in range(2)]
        self.y = [torch.zeros(T, layer.H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.graphs = [layer.capture(T, x_in=self.x[s], logits_in=self.logits[s], y_out=self.y[s])
                       for s in range(2)]
        self.up = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]

    def run(self, xs, logits, ys):
        """y_i = layer(x_i, logits_i) for pinned host tensors xs[i] [T, H] bf16,
        logits[i] [T, E] float32, into pinned host ys[i] [T, H] bf16.  Returns
        once all work is queued; the current stream waits for the last copy."""
        comp = torch.cuda.current_stream(self.layer.device)
        self.up.wait_stream(comp)
        self.down.wait_stream(comp)
        for i in range(len(xs)):
            s = i % 2
            with torch.cuda.stream(self.up):
                if i >= 2:
                    self.up.wait_event(self.computed[s])  # slot s's inputs were read by batch i - 2
                self.x[s].copy_(xs[i], non_blocking=True)
                self.logits[s].copy_(logits[i], non_blocking=True)
                self.uploaded[s].record(self.up)
            comp.wait_event(self.uploaded[s])
            if i >= 2:
                comp.wait_event(self.downloaded[s])  # slot s's output of batch i - 2 is out
            self.graphs[s].replay()
            self.computed[s].record(comp)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.computed[s])
                ys[i].copy_(self.y[s], non_blocking=True)
                self.downloaded[s].record(self.down)
        comp.wait_stream(self.up)
        comp.wait_stream(self.down)


def capture_stack(passes, x_in, y_bufs, T):
    """One CUDA graph of expert layers applied one after another to the same T
    tokens, as in a stack of decoder layers: passes = [(layer, logits), ...],
    logits [>= T, E] float32 on the device.  Pass 0 reads x_in [>= T, H]
    (bf16); pass p > 0 reads the output of pass p - 1; pass p writes
    y_bufs[p % 2].  A layer object may appear in several passes (its
    intermediate buffers are reused, the passes run in order).  Run each
    distinct layer eagerly once before capturing.  Returns (graph, y) with y
    the buffer that holds the last pass's output.
    """
    if not passes:
        raise ValueError("capture_stack needs at least one pass")
    for p, (layer, logits) in enumerate(passes):
        layer._check_io(T, x_in if p == 0 else None, logits, y_bufs[p % 2])
    dev = x_in.device
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(g, stream=side):
        x = x_in
        for p, (layer, logits) in enumerate(passes):
            y = y_bufs[p % 2]
            layer.route(logits, T)
            layer.permute(x, T)
            layer.gateup(T)
            layer.down(T)
            layer.combine(T, y)
            x = y
    torch.cuda.current_stream(dev).wait_stream(side)
    return g, y_bufs[(len(passes) - 1) % 2]
