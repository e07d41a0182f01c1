"""Seeded synthetic inputs and the named workloads of the MoE expert layer.

This module only draws random numbers and describes shapes; it holds none
of the layer's arithmetic, so the CUDA library's tests and the CPU oracle
can both be fed from it.

Workloads (the routed expert layer of Inkling 2 Small: 384 experts, top-8,
no shared expert, NVFP4 or MXFP8 experts; d_model 4096, expert ffn 2560):
  tiny_nvfp4            T=64,    H=256,  I=128,  E=8,   k=2, NVFP4
  decode_nvfp4          T=64,    H=4096, I=2560, E=384, k=8, NVFP4
  decode_mxfp8          T=256,   H=4096, I=2560, E=384, k=8, MXFP8
  prefill_nvfp4         T=8192,  H=4096, I=2560, E=384, k=8, NVFP4
  prefill_nvfp4_skewed  T=16384, H=4096, I=2560, E=384, k=8, NVFP4, Zipf bias
  prefill_mxfp8         T=8192,  H=4096, I=2560, E=384, k=8, MXFP8
  tiny_bf16_lora        T=64,    H=256,  I=128,  E=8,   k=2, BF16 + rank-32 adapters
  decode_bf16_lora      T=64,    H=4096, I=2560, E=384, k=8, BF16 + rank-32 adapters

Recipe
  x        bf16 ~ N(0, 1)            torch CPU generator, seed BASE + 2
  logits   float32 ~ N(0, 1)         torch CPU generator, seed BASE + 1
           (skewed: + 2.0 * ln(w_r), w_r = r^-1.1 / sum, r = expert + 1)
  W[e][m]  float32 ~ N(0, std^2), std = 1/sqrt(fan_in)
           (fan_in = H for gate/up, I for down), one generator per
           (expert, matrix) with seed BASE + 1000 + 3e + m, on the device
           the caller names.
  BF16     the float32 weight draws rounded to bf16; adapters A ~ N(0,
           1/fan_in), B ~ N(0, (0.15/sqrt(r))^2), rank 32, scaling 2, seed
           BASE + 500000 + 6e + m (make_expert_lora).
  s_x, s_h static float32 activation tensor scales for NVFP4, the way a
           checkpoint carries them: s_x = 8/2688 (x ~ N(0,1) stays below 8),
           s_h = 24/2688.
"""

import math
from dataclasses import dataclass

import numpy as np
import torch

BASE_SEED = 20261202

NVFP4 = "nvfp4"
MXFP8 = "mxfp8"
BF16 = "bf16"

# Adapters of the BF16 experts: rank 32 (the pages' validation run) and
# scaling alpha / rank = 2.
LORA_RANK = 32
LORA_SCALING = 2.0

S_X = np.float32(8.0 / 2688.0)
S_H = np.float32(24.0 / 2688.0)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    d_ffn: int
    num_experts: int
    top_k: int
    fmt: str
    skewed: bool = False

    @property
    def slots(self):
        return self.T * self.top_k


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_nvfp4", 64, 256, 128, 8, 2, NVFP4),
        Workload("decode_nvfp4", 64, 4096, 2560, 384, 8, NVFP4),
        Workload("decode_mxfp8", 256, 4096, 2560, 384, 8, MXFP8),
        Workload("prefill_nvfp4", 8192, 4096, 2560, 384, 8, NVFP4),
        Workload("prefill_nvfp4_skewed", 16384, 4096, 2560, 384, 8, NVFP4, skewed=True),
        # the MXFP8 layers (40-47) at the prefill batch of the NVFP4 layer
        Workload("prefill_mxfp8", 8192, 4096, 2560, 384, 8, MXFP8),
        # BF16 experts with rank-32 adapters on gate, up and down
        Workload("tiny_bf16_lora", 64, 256, 128, 8, 2, BF16),
        Workload("decode_bf16_lora", 64, 4096, 2560, 384, 8, BF16),
    ]
}


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_x(wl: Workload, seed=BASE_SEED + 2, T=None):
    """bf16 activations [T, H] ~ N(0, 1) (CPU tensor)."""
    T = wl.T if T is None else T
    x = torch.randn(T, wl.d_model, generator=_gen(seed), dtype=torch.float32)
    return x.to(torch.bfloat16)


def zipf_bias(num_experts, s=1.1, scale=2.0):
    """Per-expert logit bias 2.0 * ln(w_r), w_r = r^-s / sum_r r^-s, r = e + 1."""
    r = np.arange(1, num_experts + 1, dtype=np.float64)
    w = r ** (-s)
    w = w / w.sum()
    return (scale * np.log(w)).astype(np.float32)


def make_logits(wl: Workload, seed=BASE_SEED + 1, T=None):
    """float32 router logits [T, E] (CPU tensor)."""
    T = wl.T if T is None else T
    lg = torch.randn(T, wl.num_experts, generator=_gen(seed), dtype=torch.float32)
    if wl.skewed:
        lg = lg + torch.from_numpy(zipf_bias(wl.num_experts))[None, :]
    return lg


def weight_seed(e, m):
    return BASE_SEED + 1000 + 3 * int(e) + int(m)


def make_expert_weights(wl: Workload, e, device="cpu"):
    """float32 (W_gate [I, H], W_up [I, H], W_down [H, I]) of expert e."""
    H, I = wl.d_model, wl.d_ffn
    out = []
    for m, (rows, cols, fan_in) in enumerate(((I, H, H), (I, H, H), (H, I, I))):
        g = _gen(weight_seed(e, m), device)
        w = torch.randn(rows, cols, generator=g, dtype=torch.float32, device=device)
        out.append(w * (1.0 / math.sqrt(fan_in)))
    return tuple(out)


def make_logits_with_ties(T, E, seed):
    """Logits rounded to multiples of 0.25 in [-2, 2] so that ties are common."""
    g = _gen(seed)
    v = torch.randint(-8, 9, (T, E), generator=g).to(torch.float32) * 0.25
    return v


def make_expert_weights_bf16(wl: Workload, e, device="cpu"):
    """bf16 (W_gate [I, H], W_up [I, H], W_down [H, I]) of expert e: the
    float32 draws of make_expert_weights rounded to bf16."""
    return tuple(w.to(torch.bfloat16) for w in make_expert_weights(wl, e, device))


def make_expert_lora(wl: Workload, e, rank=LORA_RANK, device="cpu"):
    """bf16 adapters (A_gate [r, H], B_gate [I, r], A_up [r, H], B_up [I, r],
    A_down [r, I], B_down [H, r]) of expert e: A ~ N(0, 1/fan_in), B ~
    N(0, (0.15 / sqrt(r))^2), so that with scaling 2 the adapter adds about a
    third of the magnitude of the base projection.  One generator per
    (expert, matrix), seed BASE + 500000 + 6e + m."""
    H, I, r = wl.d_model, wl.d_ffn, int(rank)
    shapes = (((r, H), 1 / math.sqrt(H)), ((I, r), 0.15 / math.sqrt(r)), ((r, H), 1 / math.sqrt(H)),
              ((I, r), 0.15 / math.sqrt(r)), ((r, I), 1 / math.sqrt(I)), ((H, r), 0.15 / math.sqrt(r)))
    out = []
    for m, (shape, std) in enumerate(shapes):
        g = _gen(BASE_SEED + 500000 + 6 * int(e) + m, device)
        out.append((torch.randn(*shape, generator=g, dtype=torch.float32, device=device) * std).to(torch.bfloat16))
    return tuple(out)
