"""Integer-exact check of the tcgen05 block-scaled GEMMs (GPU).

Codes are drawn from the E2M1 value grid {0, +-0.5, ..., +-6} (for MXFP8 the
same values as E4M3 codes) and block scales from {0.5, 1, 2}; tensor scales
are 1.  Every product is a multiple of 1/16 and every partial sum stays far
below 2^24 / 16, so any summation order gives the exact result in float32:
the kernel's gate/up output must equal the float64 product bit for bit, and
its bf16 down output must equal the correctly rounded exact value.  This
pins the operand layouts, the scale-atom layout, the nibble order and the
gate/up interleave with no tolerance.  Padding rows carry random bytes,
including NaN scale codes, and must not leak into valid rows.
"""

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B
from oracle import formats as fm

from helpers import ACT_TR, encode_expert_into, kb_padded, pack_nvfp4, pad_row_bytes, swizzle_sf, sfvec, tile_matrix

GRID_E2M1 = np.array([0, 1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15], dtype=np.uint8)   # no -0
GRID_E4M3 = np.array([0x00, 0x30, 0x38, 0x3C, 0x40, 0x44, 0x48, 0x4C,
                      0xB0, 0xB8, 0xBC, 0xC0, 0xC4, 0xC8, 0xCC], dtype=np.uint8)
SF_E4M3 = np.array([0x30, 0x38, 0x40], dtype=np.uint8)       # 0.5, 1, 2
SF_E8M0 = np.array([126, 127, 128], dtype=np.uint8)          # 0.5, 1, 2


def rand_codes(rng, fmt, shape):
    g = GRID_E2M1 if fmt == "nvfp4" else GRID_E4M3
    return rng.choice(g, size=shape).astype(np.uint8)


def rand_sf(rng, fmt, shape):
    return rng.choice(SF_E4M3 if fmt == "nvfp4" else SF_E8M0, size=shape).astype(np.uint8)


def decode(fmt, codes, sf):
    v = sfvec(fmt)
    rows, K = codes.shape
    if fmt == "nvfp4":
        val = fm.e2m1_decode(codes).reshape(rows, K // v, v) * fm.e4m3_decode(sf)[..., None]
    else:
        val = fm.e4m3_decode(codes).reshape(rows, K // v, v) * fm.e8m0_decode(sf)[..., None]
    return val.reshape(rows, K)


def to_rows_bytes(fmt, codes):
    return pack_nvfp4(codes) if fmt == "nvfp4" else codes


# Expert row counts and token counts: a decode-like case (T * k <= 128 * E)
# and prefill-like ones (several 128-row blocks per expert, odd block counts,
# partly filled last blocks, an empty expert).
CASES = {
    "decode_like": (np.array([130, 0, 5, 256], dtype=np.int32), 391),
    "prefill_like": (np.array([200, 50, 300], dtype=np.int32), 550),
    "prefill_long": (np.array([300, 0, 1000], dtype=np.int32), 1300),
}

# (H, I, case): three small shapes, and the model's own d_model 4096 / expert
# ffn 2560, where the K loop turns the 4-stage ring many times (16 NVFP4 or
# 32 MXFP8 K tiles in gate/up, 10 or 20 in down), an expert spans up to 8
# row blocks and every persistent CTA walks several tiles.
SHAPES = ([(H, I, c) for H, I in [(256, 128), (512, 256), (1024, 384)] for c in ("decode_like", "prefill_like")]
          + [(4096, 2560, "decode_like"), (4096, 2560, "prefill_long")])


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
@pytest.mark.parametrize("H,I,case", SHAPES)
def test_gemm_integer_exact(cuda_device, fmt, H, I, case):
    rng = np.random.default_rng(H * 7 + I + (1 if fmt == "mxfp8" else 0) + (3 if case != "decode_like" else 0))
    counts, T = CASES[case]
    E, k = len(counts), 1
    assert (T * k > 128 * E) == (case != "decode_like")
    assert counts.sum() == T
    offsets = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
    cfg = B.make_config(E, k, H, I, fmt)
    R = B.moe_max_rows(cfg, T)
    assert R >= offsets[-1]
    v = sfvec(fmt)
    dev = cuda_device

    # weights written directly in the packed layout, tensor scales 1
    layout = B.moe_get_weights_layout(cfg)
    packed = np.zeros(layout.total_bytes, dtype=np.uint8)
    W = {}
    for e in range(E):
        q = {}
        for m, (rows, K) in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I))):
            q[m] = (rand_codes(rng, fmt, (rows, K)), rand_sf(rng, fmt, (rows, K // v)), np.float32(1.0))
        encode_expert_into(packed, layout, fmt, e, H, I, q)
        W[e] = {m: decode(fmt, q[m][0], q[m][1]) for m in q}

    # activations: valid rows from the grid, padding rows random bytes
    bpe = 4 if fmt == "nvfp4" else 8
    a_codes = rng.integers(0, 256, (R, kb_padded(H, fmt)), dtype=np.uint8)
    a_sf = rng.integers(0, 256, (R, H // v), dtype=np.uint8)
    A = np.zeros((R, H))
    for e in range(E):
        lo, c = offsets[e], counts[e]
        if c == 0:
            continue
        codes = rand_codes(rng, fmt, (c, H))
        sf = rand_sf(rng, fmt, (c, H // v))
        a_codes[lo:lo + c, :H * bpe // 8] = to_rows_bytes(fmt, codes)
        a_sf[lo:lo + c] = sf
        A[lo:lo + c] = decode(fmt, codes, sf)

    t = lambda a, dt=torch.uint8: torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(dev)
    d_packed = t(packed)
    d_a = t(tile_matrix(a_codes, ACT_TR))
    d_asf = t(swizzle_sf(a_sf))
    d_off = t(offsets, torch.int32)
    d_cnt = t(counts, torch.int32)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    scale = one if fmt == "nvfp4" else None
    h_codes = torch.zeros(B.moe_codes_bytes(cfg, R, I), dtype=torch.uint8, device=dev)
    h_sf = torch.zeros(B.moe_sf_bytes(cfg, R, I), dtype=torch.uint8, device=dev)
    dbg = torch.full((R, 2 * I), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B.moe_forward_gateup(cfg, T, d_packed, d_a, d_asf, scale, scale, d_off, d_cnt, h_codes, h_sf, dbg, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = dbg.cpu().numpy()
    for e in range(E):
        lo, c = offsets[e], counts[e]
        if c == 0:
            continue
        g = A[lo:lo + c] @ W[e]["gate"].T
        u = A[lo:lo + c] @ W[e]["up"].T
        assert np.all(np.abs(g) < 2 ** 20)
        np.testing.assert_array_equal(got[lo:lo + c, :I], g.astype(np.float32), err_msg=f"gate e={e}")
        np.testing.assert_array_equal(got[lo:lo + c, I:], u.astype(np.float32), err_msg=f"up e={e}")
    # rows without a slot are never written
    valid = np.zeros(R, dtype=bool)
    for e in range(E):
        valid[offsets[e]:offsets[e] + counts[e]] = True
    assert np.all(np.isnan(got[~valid]))

    # down GEMM on intermediate codes chosen the same way
    hc = rng.integers(0, 256, (R, kb_padded(I, fmt)), dtype=np.uint8)
    hs = rng.integers(0, 256, (R, I // v), dtype=np.uint8)
    Hm = np.zeros((R, I))
    for e in range(E):
        lo, c = offsets[e], counts[e]
        if c == 0:
            continue
        codes = rand_codes(rng, fmt, (c, I))
        sf = rand_sf(rng, fmt, (c, I // v))
        hc[lo:lo + c, :I * bpe // 8] = to_rows_bytes(fmt, codes)
        hs[lo:lo + c] = sf
        Hm[lo:lo + c] = decode(fmt, codes, sf)
    out = torch.full((R, H), float("nan"), dtype=torch.bfloat16, device=dev)
    B.moe_forward_down(cfg, T, d_packed, t(tile_matrix(hc, ACT_TR)), t(swizzle_sf(hs)), scale, d_off, d_cnt, out,
                       status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o = out.float().cpu().numpy().astype(np.float64)
    for e in range(E):
        lo, c = offsets[e], counts[e]
        if c == 0:
            continue
        ref = fm.bf16_round(Hm[lo:lo + c] @ W[e]["down"].T)
        np.testing.assert_array_equal(o[lo:lo + c], ref, err_msg=f"down e={e}")
    assert np.all(np.isnan(o[~valid]))
