"""Benchmark of the routed MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--only] [--impl ours|reference]

One step is one pass of the whole layer over one batch of synthetic inputs
already resident in HBM: route -> permute+quantize -> gate/up GEMM (SwiGLU +
requantization) -> down GEMM -> weighted combine.  Default workload: the
largest single-GPU layer, NVFP4 with Zipf-skewed routing (16,384 tokens,
d_model 4096, expert ffn 2560, 384 experts, top-8); on one GPU the same run
also measures the other four full-size layers (decode NVFP4 T=64, decode
MXFP8 T=256, prefill NVFP4 T=8192, prefill MXFP8 T=8192) and reports them
under "workloads" (--only skips them).  Weights are random-init of that
architecture, quantized once by the library before timing.  Every timed step
is bracketed by CUDA events on the launching stream; L2 is flushed (a 512 MiB
write) between timed steps, outside the events.  With --gpus N > 1 (launched by torchrun) every rank runs
an independent replica of the same workload (the layer has no data-path
exchange on one node: "replicas only"), the times are max-reduced over ranks
and `value` counts the tokens of all ranks.

--impl reference times the CPU oracle (oracle/, numpy) on a bounded sample of
the same workload on the host cores; under torchrun only rank 0 runs it.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_moe_expert_top_b200 import inputs  # noqa: E402

METRIC = "MoE layer tokens/s on 1 B200; % of HBM or NVFP4/FP8 tensor roofline"
UNIT = "tokens/s"
# the largest single-GPU layer, and the other full-size layers measured beside it
HEADLINE = "prefill_nvfp4_skewed"
FULL_SIZE = ("decode_nvfp4", "decode_mxfp8", "prefill_nvfp4", "prefill_nvfp4_skewed", "prefill_mxfp8",
             "decode_bf16_lora")


# --------------------------------------------------------------------------- helpers

def pct(values, q):
    """q-th percentile (linear interpolation) of a non-empty list."""
    return float(np.percentile(np.asarray(values, dtype=np.float64), q))


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, world_size, device=None):
    """Element-wise max of a list of floats over all ranks (identity for one rank)."""
    if world_size <= 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world_size):
    if world_size > 1:
        import torch.distributed as dist
        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """SM clock and throttle-reason samples during the timed region.

    NVML is polled from a thread every ~2 ms (the timed regions of the short
    layers last a few tens of milliseconds); start() returns once the first
    sample is in.  Falls back to `nvidia-smi -lms` when NVML is unavailable.
    Only reads the GPU's state.
    """

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80), ("gpu_idle", 0x1),
               ("applications_clocks_setting", 0x2), ("sync_boost", 0x10), ("display_clock_setting", 0x100))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.thread = None
        self.proc = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except pynvml.NVMLError:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
        except Exception:  # no NVML: nvidia-smi at its shortest interval
            self._start_smi()
            return
        self.stop_flag = threading.Event()
        first = threading.Event()
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

        def run():
            while True:
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), max_mhz,
                                         nv.nvmlDeviceGetCurrentClocksEventReasons(h),
                                         nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except nv.NVMLError:
                    pass
                first.set()
                if self.stop_flag.wait(0.002):
                    break

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        first.wait(5.0)

    def _start_smi(self):
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            samples = self.samples
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            samples = []
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        mask = sum(bit for (_, bit), v in zip(self.REASONS[:4], parts[5:9])
                                   if v.lower().startswith("active"))
                        samples.append((float(parts[1]), float(parts[2]), mask, float(parts[3])))
                    except ValueError:
                        continue
            os.unlink(self.path)
        else:
            return None
        if not samples:
            return None
        reasons = sorted({n for s_ in samples for n, bit in self.REASONS if s_[2] & bit})
        clk = [s_[0] for s_ in samples]
        return {"sm_mhz": statistics.median(clk), "sm_max_mhz": max(s_[1] for s_ in samples),
                "sm_mhz_min": min(clk), "sm_mhz_max_seen": max(clk),
                "power_w_max": round(max(s_[3] for s_ in samples), 1), "reasons": reasons, "samples": len(samples),
                "source": "nvml, 2 ms" if self.thread is not None else "nvidia-smi, 50 ms"}


# --------------------------------------------------------------------------- workload

def build_layer(wl, device, T):
    from fp8_moe_expert_top_b200.layer import ExpertLayer
    layer = ExpertLayer(wl.num_experts, wl.top_k, wl.d_model, wl.d_ffn, wl.fmt, T, device,
                        s_x=inputs.S_X, s_h=inputs.S_H)
    chunk = 16
    for e0 in range(0, wl.num_experts, chunk):
        n = min(chunk, wl.num_experts - e0)
        if wl.fmt == inputs.BF16:
            # bf16 weights with rank-32 adapters on gate, up and down
            ws = [inputs.make_expert_weights_bf16(wl, e, device=device) for e in range(e0, e0 + n)]
            ls = [inputs.make_expert_lora(wl, e, device=device) for e in range(e0, e0 + n)]
            lora = tuple(torch.stack([l_[m] for l_ in ls]).contiguous() for m in range(6))
            layer.pack_experts_bf16(e0, *(torch.stack([w[m] for w in ws]).contiguous() for m in range(3)),
                                    lora=lora, lora_rank=inputs.LORA_RANK, lora_scaling=inputs.LORA_SCALING)
            del ws, ls, lora
            continue
        ws = [inputs.make_expert_weights(wl, e, device=device) for e in range(e0, e0 + n)]
        wg = torch.stack([w[0] for w in ws]).contiguous()
        wu = torch.stack([w[1] for w in ws]).contiguous()
        wd = torch.stack([w[2] for w in ws]).contiguous()
        layer.quantize_experts(e0, wg, wu, wd)
        del ws, wg, wu, wd
    torch.cuda.synchronize()
    return layer


def phase_bytes(wl, n_touched, slots):
    """Algorithmic HBM bytes of each phase (compulsory traffic, no re-reads)."""
    H, I, E, T = wl.d_model, wl.d_ffn, wl.num_experts, wl.T
    if wl.fmt == inputs.BF16:
        # bf16 weights; each row carries its adapter's 64-element tile (B),
        # plus the adapters' A (64 rows of H and of I per expert)
        q = 2.0
        w13 = n_touched * (2 * I * (H + 64) + 64 * H) * 2
        w2 = n_touched * (H * (I + 64) + 64 * I) * 2
    else:
        bpe = 0.5 if wl.fmt == inputs.NVFP4 else 1.0
        sf = 1.0 / (16 if wl.fmt == inputs.NVFP4 else 32)
        q = bpe + sf                              # bytes per quantized element (codes + block scales)
        w13 = n_touched * 2 * I * H * q
        w2 = n_touched * H * I * q
    return {
        "route": T * E * 4 + T * wl.top_k * 8,
        "permute": T * H * 2 + slots * H * q,
        "gateup": w13 + slots * H * q + slots * I * q,
        "down": w2 + slots * I * q + slots * H * 2,
        "combine": slots * H * 2 + T * H * 2 + T * wl.top_k * 8,
        "layer": w13 + w2 + T * H * 2 + T * E * 4 + T * H * 2,
    }


PHASES = ("route", "permute", "gateup", "down", "combine")


def kernels_per_step(wl, T):
    """The library's kernel launches in one layer step: routing (top-k, then
    scan and scatter, or for batches of up to 512 tokens with at most 8192
    bitmap words one small-batch kernel), permute, gate/up (BF16: with the
    two adapter shrinks before and after it), down, combine."""
    W = (T + 31) // 32
    small = 0 < T <= 512 and wl.num_experts <= 1024 and wl.num_experts * W <= 8192
    route = 2 if small else 3
    gateup = 3 if wl.fmt == inputs.BF16 else 1
    return route + 1 + gateup + 1 + 1


def run_ours(args, wl, ws, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    T = wl.T
    layer = build_layer(wl, device, T)
    x_h = inputs.make_x(wl)
    lg_h = inputs.make_logits(wl)
    x = x_h.to(device)
    lg = lg_h.to(device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        layer.route(lg, T)
        if ev is not None:
            ev[1].record(stream)
        layer.permute(x, T)
        if ev is not None:
            ev[2].record(stream)
        layer.gateup(T)
        if ev is not None:
            ev[3].record(stream)
        layer.down(T)
        if ev is not None:
            ev[4].record(stream)
        layer.combine(T)
        if ev is not None:
            ev[5].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    counts = layer.expert_counts.cpu().numpy()
    n_touched = int((counts > 0).sum())
    slots = T * wl.top_k
    status = int(layer.status.item())
    if status != 0:
        raise RuntimeError(f"device status word {status:#x} after warm-up")

    # eager steps (five host calls per step), for reference
    eager_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step(eager_ev[i])
    torch.cuda.synchronize()
    eager_ms = sum(ev[0].elapsed_time(ev[5]) for ev in eager_ev) / args.steps

    # the timed region: the layer captured once as a CUDA graph, replayed per step
    gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
    layer.x_in = x.clone()
    layer.logits_in = lg.clone()
    graph = layer.capture(T, events=gev)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    per_phase = {p: [] for p in PHASES}
    step_ms = []
    barrier(ws)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()                      # L2 flush, outside the events
        graph.replay()
        torch.cuda.synchronize()
        for j, p in enumerate(PHASES):
            per_phase[p].append(gev[j].elapsed_time(gev[j + 1]))
        step_ms.append(gev[0].elapsed_time(gev[5]))
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status word {int(layer.status.item()):#x} after the timed steps")
    total_ms = sum(step_ms)
    total_ms = max_over_ranks([total_ms], ws, device)[0]

    # end to end through the public API: pinned host inputs in, host output
    # back, every step; the host copies of neighbouring steps overlap the
    # layer (HostPipeline).  No L2 flush here: each step streams the touched
    # experts' weights (GBs), far more than L2.
    from fp8_moe_expert_top_b200.layer import HostPipeline
    x_pin = x_h.pin_memory()
    lg_pin = lg_h.pin_memory()
    y_pins = [torch.empty(T, wl.d_model, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe = HostPipeline(layer, T)
    n_warm = max(2, args.warmup)
    pipe.run([x_pin] * n_warm, [lg_pin] * n_warm, [y_pins[i % 2] for i in range(n_warm)])
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.run([x_pin] * args.steps, [lg_pin] * args.steps, [y_pins[i % 2] for i in range(args.steps)])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], ws, device)[0]
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status word {int(layer.status.item()):#x} after the end-to-end steps")
    del pipe
    del graph

    # roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    bytes_ = phase_bytes(wl, n_touched, slots)
    mean_ms = {p: statistics.mean(v) for p, v in per_phase.items()}
    dom = max(("gateup", "down"), key=lambda p: mean_ms[p])
    flops_slot = 6.0 * wl.d_model * wl.d_ffn
    dom_flops = slots * flops_slot * (2.0 / 3.0 if dom == "gateup" else 1.0 / 3.0)
    t_dom = mean_ms[dom] * 1e-3
    bf16 = peaks.get("bf16_tflops", 1590.0)
    ratio = {inputs.NVFP4: 4.0, inputs.MXFP8: 2.0, inputs.BF16: 1.0}[wl.fmt]   # nominal fp4 / fp8 : bf16
    tensor_peak = bf16 * ratio
    t_hbm = bytes_[dom] / (peaks["hbm_gbs"] * 1e9)
    t_tc = dom_flops / (tensor_peak * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": bytes_[dom] / t_dom / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": dom_flops / t_dom / 1e12, "peak": tensor_peak, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # against the nominal B200 peaks (8 TB/s HBM; 9 / 4.5 PFLOP/s dense NVFP4 / FP8)
    nominal_tensor = {inputs.NVFP4: 9000.0, inputs.MXFP8: 4500.0, inputs.BF16: 2250.0}[wl.fmt]
    roof["frac_nominal"] = roof["achieved"] / (8000.0 if roof["bound"] == "hbm" else nominal_tensor)
    roof["kernel"] = f"moe_gemm_kernel ({dom})"
    roof["peak_source"] = peak_kind + (" hbm_gbs" if roof["bound"] == "hbm" else
                                       f" bf16_tflops x {ratio:g} (nominal ratio)")
    roof["traffic"] = measured_traffic(wl.name, dom)
    # whole-layer roofline (slower of bytes at HBM peak and FLOPs at tensor peak)
    layer_t = max(bytes_["layer"] / (peaks["hbm_gbs"] * 1e9), slots * flops_slot / (tensor_peak * 1e12))
    # nominal B200 peaks for context: 8 TB/s HBM, 9 / 4.5 / 2.25 PFLOP/s dense NVFP4 / FP8 / BF16
    layer_t_nominal = max(bytes_["layer"] / 8.0e12, slots * flops_slot / (nominal_tensor * 1e12))
    value = ws * T * args.steps / (total_ms * 1e-3)
    out = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.fmt,
        "data": "synthetic (seeded N(0,1) x and logits, N(0,1/fan_in) weights, random init)",
        "config": {"workload": wl.name, "T": T, "d_model": wl.d_model, "d_ffn": wl.d_ffn,
                   "num_experts": wl.num_experts, "top_k": wl.top_k, "format": wl.fmt,
                   "experts_touched": n_touched, "l2": "flushed between timed steps (512 MiB write)",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "roofline": roof,
        "layer_roofline_frac": layer_t / (total_ms * 1e-3 / args.steps),
        "layer_roofline_frac_nominal": layer_t_nominal / (total_ms * 1e-3 / args.steps),
        "step_ms_pct": {"p10": pct(step_ms, 10), "p50": pct(step_ms, 50), "p90": pct(step_ms, 90)},
        "phase_ms": {p: round(mean_ms[p], 4) for p in PHASES},
        "eager_ms_per_step": eager_ms,
        "timing": "CUDA graph of the five calls replayed per step; external CUDA events between the steps",
        "e2e": {"value": ws * T * args.steps / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": int(x_h.numel() * 2 + lg_h.numel() * 4),
                "d2h_bytes_per_step": int(T * wl.d_model * 2),
                "overlap": "HostPipeline: step i+1's upload and step i-1's download overlap step i "
                           "(two graphs, upload and download streams); no L2 flush, each step streams "
                           "GBs of weights"},
        "gpu_launches": kernels_per_step(wl, T) * args.steps,
        "clocks": clk,
    }
    return out, layer


def time_fused_router(args, device):
    """Routing from the layer input (router scores fused with the top-k,
    moe_router_topk) against the unfused pair (the router product by a
    library bf16 GEMM into float32 logits, then moe_route_topk) and against
    routing from given logits alone (moe_route_topk, no router product), at
    the decode, prefill and skewed batch sizes.  Each is one CUDA graph,
    replayed args.steps times with an L2 flush between replays; per-replay
    device time from CUDA events."""
    from fp8_moe_expert_top_b200 import binding as B
    torch.cuda.set_device(device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    out = {}
    for name in ("decode_nvfp4", "prefill_nvfp4", "prefill_nvfp4_skewed"):
        wl = inputs.WORKLOADS[name]
        T, E, H, k = wl.T, wl.num_experts, wl.d_model, wl.top_k
        cfg = B.make_config(E, k, H, wl.d_ffn, wl.fmt)
        R = B.moe_max_rows(cfg, T)
        i32 = dict(dtype=torch.int32, device=device)
        bufs = (torch.empty(T, k, **i32), torch.empty(T, k, dtype=torch.float32, device=device),
                torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R, **i32), torch.empty(T * k, **i32))
        ws = torch.empty(B.moe_route_workspace_bytes(cfg, T), dtype=torch.uint8, device=device)
        x = inputs.make_x(wl).to(device)
        lg = inputs.make_logits(wl).to(device)
        g = torch.Generator(device=device)
        g.manual_seed(inputs.BASE_SEED + 3)
        w_r = (torch.randn(E, H, generator=g, device=device) / H ** 0.5).to(torch.bfloat16)
        status = torch.zeros(1, **i32)
        lg_mm = torch.empty(T, E, dtype=torch.float32, device=device)

        def gemm_then_route():
            # timing baseline only: a library bf16 GEMM (bf16 result, widened
            # to float32 logits), then routing from those logits
            lg_mm.copy_(torch.mm(x, w_r.t()))
            B.moe_route_topk(cfg, T, lg_mm, *bufs, ws)

        calls = {"from_logits": lambda: B.moe_route_topk(cfg, T, lg, *bufs, ws),
                 "gemm_then_route": gemm_then_route,
                 "fused_router": lambda: B.moe_router_topk(cfg, T, x, w_r, None, *bufs, ws, status)}
        res = {}
        for key, fn in calls.items():
            for _ in range(args.warmup):
                fn()
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(device=device)
            side.wait_stream(stream)
            with torch.cuda.graph(graph, stream=side):
                fn()
            stream.wait_stream(side)
            times = []
            for _ in range(args.steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            res[key + "_ms"] = statistics.mean(times)
            del graph
        if int(status.item()) != 0:
            raise RuntimeError(f"device status word {int(status.item()):#x} from the fused router")
        flops = 2.0 * T * E * H
        res["router_tflops"] = flops / (res["fused_router_ms"] * 1e-3) / 1e12
        res["fused_vs_gemm_then_route"] = res["gemm_then_route_ms"] / res["fused_router_ms"]
        res["T"] = T
        out[name] = res
    return out


def measured_traffic(workload, phase):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel source
    has not changed since it was captured (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(workload, {}).get(phase)
    if not ent:
        return None
    if ent.get("gemm_sha") != gemm_source_sha():
        return None
    return ent.get("bytes")


def gemm_source_sha():
    """Hash of the sources the one-SM GEMM kernel is compiled from."""
    h = hashlib.sha256()
    for f in ("gemm.cu", "gemm_common.cuh", "common.cuh", "quant.cuh"):
        with open(os.path.join(ROOT, "fp8_moe_expert_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------- expert stack

def run_depth(args, local, n_nv, n_mx):
    """The expert layers of the whole model depth applied to one batch: n_nv
    NVFP4 passes then n_mx MXFP8 passes, each fed the previous pass's output
    and its own seeded logits (the router is outside the layer), captured as
    one CUDA graph.  Two weight sets (one NVFP4 and one MXFP8 layer, each larger
    than L2) serve all passes, so every pass streams its weights from HBM."""
    import dataclasses
    from fp8_moe_expert_top_b200.layer import capture_stack
    T = args.tokens if args.tokens is not None else 64
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl_n = dataclasses.replace(inputs.WORKLOADS["decode_nvfp4"], T=T)
    wl_m = dataclasses.replace(inputs.WORKLOADS["decode_mxfp8"], T=T)
    ln, lm = build_layer(wl_n, device, T), build_layer(wl_m, device, T)
    passes = []
    for p in range(n_nv + n_mx):
        wl = wl_n if p < n_nv else wl_m
        passes.append((ln if p < n_nv else lm, wl,
                       inputs.make_logits(wl, seed=inputs.BASE_SEED + 100 + p).to(device)))
    x = inputs.make_x(wl_n).to(device)
    # eager pass: sets up every kernel and gives each pass's touched experts
    layer_bytes, cur = 0.0, x
    for layer, wl, lg in passes:
        cur = layer.forward(cur, lg).clone()
        n_touched = int((layer.expert_counts.cpu() > 0).sum())
        layer_bytes += phase_bytes(wl, n_touched, T * wl.top_k)["layer"]
    y_bufs = [torch.zeros(T, wl_n.d_model, dtype=torch.bfloat16, device=device) for _ in range(2)]
    graph, _ = capture_stack([(l, lg) for l, _, lg in passes], x, y_bufs, T)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    clocks = ClockSampler(local)
    clocks.start()
    step_ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    clk = clocks.stop()
    for layer in (ln, lm):
        if int(layer.status.item()) != 0:
            raise RuntimeError(f"device status word {int(layer.status.item()):#x}")
    peaks, _ = load_peaks()
    ms = statistics.mean(step_ms)
    return {
        "metric": f"expert-layer stack ({n_nv} NVFP4 + {n_mx} MXFP8 layers) tokens/s on 1 B200",
        "value": T / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4+mxfp8",
        "data": "synthetic (seeded N(0,1) x and per-layer logits, N(0,1/fan_in) weights, random init)",
        "config": {"workload": f"expert_stack_{n_nv}x_nvfp4_{n_mx}x_mxfp8_t{T}", "T": T, "d_model": wl_n.d_model,
                   "d_ffn": wl_n.d_ffn, "num_experts": wl_n.num_experts, "top_k": wl_n.top_k,
                   "l2": "flushed between timed steps (512 MiB write)", "parallelism": "single GPU"},
        "stack_roofline_frac": (layer_bytes / (peaks["hbm_gbs"] * 1e9)) / (ms * 1e-3),
        "ms_per_layer": ms / (n_nv + n_mx),
        "step_ms_pct": {"p10": pct(step_ms, 10), "p50": pct(step_ms, 50), "p90": pct(step_ms, 90)},
        "gpu_launches": (n_nv * kernels_per_step(wl_n, T) + n_mx * kernels_per_step(wl_m, T)) * args.steps,
        "clocks": clk,
    }


# --------------------------------------------------------------------------- CPU oracle

def _oracle_quantize(args_):
    e, fmt, wg, wu, wd = args_
    from oracle import moe as omoe
    return e, omoe.quantize_expert(wg, wu, wd, fmt)


def oracle_sample(wl, n_tokens):
    """Inputs of the bounded oracle sample: the first n_tokens tokens and the
    quantized weights of every expert they select (prepared outside timing,
    in a spawn pool).  Weights are drawn on the GPU when there is one, as the
    library's benchmark does, else on the CPU."""
    import multiprocessing as mp
    from oracle import route as ort
    x = inputs.make_x(wl)[:n_tokens].float().numpy()
    lg = inputs.make_logits(wl)[:n_tokens].numpy()
    ids = ort.topk_select(lg, wl.top_k)
    need = sorted(set(int(e) for e in ids.reshape(-1)))
    wdev = "cuda" if torch.cuda.is_available() else "cpu"
    jobs = []
    for e in need:
        wg, wu, wd = (w.cpu().numpy() for w in inputs.make_expert_weights(wl, e, device=wdev))
        jobs.append((e, wl.fmt, wg, wu, wd))
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(len(need), max(1, os.cpu_count() or 1))) as pool:
        experts = dict(pool.map(_oracle_quantize, jobs))
    return x, lg, experts


def time_oracle(wl, x, lg, experts):
    from oracle import moe as omoe
    t0 = time.perf_counter()
    omoe.forward_tokens(x, lg, experts, wl.top_k, wl.fmt, inputs.S_X, inputs.S_H)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return 1


def default_sample_tokens(wl):
    return 2 if wl.d_model * wl.d_ffn > (1 << 20) else min(wl.T, 64)


def cpu_baseline(wl, n_tokens=None):
    n = n_tokens or default_sample_tokens(wl)
    x, lg, experts = oracle_sample(wl, n)
    dt = time_oracle(wl, x, lg, experts)
    return {"value": n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} tokens of {wl.name} (their {len(experts)} experts' weights quantized by the "
                      f"oracle beforehand, untimed); numpy float64, host cpu_count={os.cpu_count()}"}


def run_reference(args, wl, ws, rank):
    if rank != 0:
        return None
    # one token per step at full size (about 4 s of host work each), so a
    # run of the default 20 + 5 steps ends within a few minutes
    n = 1 if wl.d_model * wl.d_ffn > (1 << 20) else default_sample_tokens(wl)
    x, lg, experts = oracle_sample(wl, n)
    for _ in range(args.warmup):
        time_oracle(wl, x, lg, experts)
    times = [time_oracle(wl, x, lg, experts) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    cores = blas_threads()
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) x and logits, N(0,1/fan_in) weights, random init)",
        "config": {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "d_ffn": wl.d_ffn,
                   "num_experts": wl.num_experts, "top_k": wl.top_k, "format": wl.fmt,
                   "sample_tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} tokens of {wl.name} per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--only", action="store_true", help="measure only --workload, not the other full-size layers")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--router-only", action="store_true",
                    help="time only routing: the fused router against routing from given logits")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling only: override the number of experts (smaller device footprint for ncu)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling only: override the number of tokens (with --experts, keeps rows per expert)")
    ap.add_argument("--depth", default=None, metavar="N_NVFP4,N_MXFP8",
                    help="time the expert layers of a whole model depth on one batch (e.g. 40,8), "
                         "--tokens tokens (default 64)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = inputs.WORKLOADS[args.workload]
    if args.experts is not None or args.tokens is not None:
        import dataclasses
        if args.experts is not None:
            wl = dataclasses.replace(wl, name=f"{wl.name}_e{args.experts}", num_experts=args.experts)
        if args.tokens is not None:
            wl = dataclasses.replace(wl, name=f"{wl.name}_t{args.tokens}", T=args.tokens)
    ws, rank, local = dist_env()
    if ws != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {ws}", file=sys.stderr)
    if args.depth is not None:
        if ws > 1 or args.impl != "ours":
            ap.error("--depth runs the library on one GPU")
        n_nv, n_mx = (int(v) for v in args.depth.split(","))
        print(json.dumps(run_depth(args, local, n_nv, n_mx)))
        return 0
    if args.impl == "reference":
        out = run_reference(args, wl, ws, rank)
        if out is not None:
            print(json.dumps(out))
        return 0
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.router_only:
            if rank == 0:
                print(json.dumps({"fused_router": time_fused_router(args, torch.device("cuda", local))}))
            return 0
        out, layer = run_ours(args, wl, ws, rank, local)
        del layer
        torch.cuda.empty_cache()
        if ws == 1 and not args.only and args.experts is None and args.tokens is None:
            out["workloads"] = {}
            for name in FULL_SIZE:
                if name == wl.name:
                    continue
                o, layer = run_ours(args, inputs.WORKLOADS[name], ws, rank, local)
                del layer
                torch.cuda.empty_cache()
                out["workloads"][name] = {key: o[key] for key in (
                    "value", "unit", "ms_per_step", "dtype", "config", "roofline", "layer_roofline_frac",
                    "layer_roofline_frac_nominal", "step_ms_pct", "phase_ms", "e2e", "gpu_launches", "clocks")}
            out["fused_router"] = time_fused_router(args, torch.device("cuda", local))
        if rank == 0:
            if ws == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(wl)
            print(json.dumps(out))
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
