"""Test-side decoding of the library's buffer layouts into plain arrays.

Written from the layout contract of include/moe_b200.h (not from the CUDA
code): a code row holds K codes (NVFP4 element 2i in the low nibble of byte
i), padded to kb = a multiple of 128 bytes; code matrices are stored as tiles
of TR rows x 128 bytes (TR = 256 for weights, 128 for activations), K tile
fastest, and inside a tile row r's 16-byte chunk c sits at r * 128 +
(c ^ (r % 8)) * 16; block scales in 512-byte atoms of 128 rows x 4 columns,
K direction fastest, byte (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4 inside
an atom; w13 rows interleave gate and up channels in groups of 32.
"""

import numpy as np


def sf_index(rows, nsf):
    """Byte offset of every (row, col) scale, as an int64 array [rows, nsf]."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    c = np.arange(nsf, dtype=np.int64)[None, :]
    atom = (r // 128) * (nsf // 4) + c // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4


def sf_index_rows(rows, nsf):
    """Byte offset of every (row, col) scale of the given rows, int64 [len(rows), nsf]."""
    r = np.asarray(rows, dtype=np.int64)[:, None]
    c = np.arange(nsf, dtype=np.int64)[None, :]
    atom = (r // 128) * (nsf // 4) + c // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4


def unswizzle_sf(buf, rows, nsf):
    """[rows, nsf] uint8 scales from an atom-layout buffer (rows % 128 == 0)."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    return buf[sf_index(rows, nsf)]


def swizzle_sf(sf):
    """Atom-layout bytes of a [rows, nsf] scale matrix (rows % 128 == 0)."""
    rows, nsf = sf.shape
    out = np.zeros(rows * nsf, dtype=np.uint8)
    out[sf_index(rows, nsf)] = sf
    return out


WEIGHT_TR = 256
ACT_TR = 128


def kb_padded(K, fmt):
    bits = 4 if fmt == "nvfp4" else 8
    return (K * bits // 8 + 127) // 128 * 128


def tile_offsets(rows, kb, TR):
    """Byte offset of every (row, byte) of the given rows in a tiled code matrix."""
    r_all = np.asarray(rows, dtype=np.int64)[:, None]
    b = np.arange(kb, dtype=np.int64)[None, :]
    tile = (r_all // TR) * (kb // 128) + b // 128
    r = r_all % TR
    bb = b % 128
    return tile * TR * 128 + r * 128 + ((bb // 16) ^ (r % 8)) * 16 + bb % 16


def untile_rows(buf, rows, kb, TR):
    """[len(rows), kb] bytes of the given rows of a tiled code matrix."""
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[tile_offsets(rows, kb, TR)]


def tile_matrix(mat, TR):
    """Tiled bytes of a [rows, kb] byte matrix (rows % TR == 0, kb % 128 == 0)."""
    rows, kb = mat.shape
    out = np.zeros(rows * kb, dtype=np.uint8)
    out[tile_offsets(np.arange(rows), kb, TR)] = mat
    return out


def pad_row_bytes(mat, kb):
    rows, n = mat.shape
    out = np.zeros((rows, kb), dtype=np.uint8)
    out[:, :n] = mat
    return out


def unpack_nvfp4(codes_bytes, rows, K):
    """[rows, K] 4-bit codes from packed bytes [rows, K/2]."""
    b = np.asarray(codes_bytes, dtype=np.uint8).reshape(rows, K // 2)
    out = np.empty((rows, K), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def pack_nvfp4(codes):
    rows, K = codes.shape
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(fmt, row_bytes, rows, K):
    """[rows, K] codes from [rows, >= K*bits/8] code-row bytes."""
    b = np.asarray(row_bytes, dtype=np.uint8).reshape(rows, -1)
    if fmt == "nvfp4":
        return unpack_nvfp4(np.ascontiguousarray(b[:, :K // 2]), rows, K)
    return np.ascontiguousarray(b[:, :K])


def tiled_codes(fmt, buf, rows, K, TR):
    """[len(rows), K] codes of the given rows of a tiled code buffer."""
    rows = np.asarray(rows, dtype=np.int64)
    return unpack_codes(fmt, untile_rows(buf, rows, kb_padded(K, fmt), TR), len(rows), K)


def sfvec(fmt):
    return 16 if fmt == "nvfp4" else 32


def w13_row(m, c):
    """Row of w13 holding channel c of gate (m = 0) or up (m = 1)."""
    c = np.asarray(c)
    return 64 * (c // 32) + 32 * m + c % 32


def decode_expert(packed, layout, fmt, e, H, I):
    """(codes, scales, tensor scale) of gate, up and down of expert e.

    packed: uint8 numpy array of the whole packed buffer (or a copy of it),
    or a function (offset, nbytes) -> uint8 numpy array of that byte range.
    """
    v = sfvec(fmt)
    if callable(packed):
        get = packed
    else:
        p = np.asarray(packed, dtype=np.uint8)
        get = lambda off, n: p[off:off + n]  # noqa: E731
    kb13, kb2 = kb_padded(H, fmt), kb_padded(I, fmt)
    n13 = 2 * I * kb13
    c13 = get(layout.w13_codes + e * n13, n13)
    s13n = 2 * I * H // v
    s13 = get(layout.w13_sf + e * s13n, s13n)
    n2 = H * kb2
    c2 = get(layout.w2_codes + e * n2, n2)
    s2n = H * I // v
    s2 = get(layout.w2_sf + e * s2n, s2n)
    scales = np.ascontiguousarray(get(layout.scales + 12 * e, 12)).view(np.float32)
    codes13 = tiled_codes(fmt, c13, np.arange(2 * I), H, WEIGHT_TR)
    sf13 = unswizzle_sf(s13, 2 * I, H // v)
    codes2 = tiled_codes(fmt, c2, np.arange(H), I, WEIGHT_TR)
    sf2 = unswizzle_sf(s2, H, I // v)
    gi, ui = w13_row(0, np.arange(I)), w13_row(1, np.arange(I))
    return {
        "gate": (codes13[gi], sf13[gi], np.float32(scales[0])),
        "up": (codes13[ui], sf13[ui], np.float32(scales[1])),
        "down": (codes2, sf2, np.float32(scales[2])),
    }


def encode_expert_into(packed, layout, fmt, e, H, I, q):
    """Write expert e's (codes, scales, tensor scale) triples into packed (numpy)."""
    v = sfvec(fmt)
    kb13, kb2 = kb_padded(H, fmt), kb_padded(I, fmt)
    codes13 = np.zeros((2 * I, H), dtype=np.uint8)
    sf13 = np.zeros((2 * I, H // v), dtype=np.uint8)
    gi, ui = w13_row(0, np.arange(I)), w13_row(1, np.arange(I))
    codes13[gi], sf13[gi] = q["gate"][0], q["gate"][1]
    codes13[ui], sf13[ui] = q["up"][0], q["up"][1]
    raw13 = pad_row_bytes(pack_nvfp4(codes13) if fmt == "nvfp4" else codes13, kb13)
    n13 = 2 * I * kb13
    packed[layout.w13_codes + e * n13: layout.w13_codes + (e + 1) * n13] = tile_matrix(raw13, WEIGHT_TR)
    s13n = 2 * I * H // v
    packed[layout.w13_sf + e * s13n: layout.w13_sf + (e + 1) * s13n] = swizzle_sf(sf13)
    c2 = q["down"][0]
    raw2 = pad_row_bytes(pack_nvfp4(c2) if fmt == "nvfp4" else c2, kb2)
    n2 = H * kb2
    packed[layout.w2_codes + e * n2: layout.w2_codes + (e + 1) * n2] = tile_matrix(raw2, WEIGHT_TR)
    s2n = H * I // v
    packed[layout.w2_sf + e * s2n: layout.w2_sf + (e + 1) * s2n] = swizzle_sf(q["down"][1])
    sc = np.array([q["gate"][2], q["up"][2], q["down"][2]], dtype=np.float32)
    packed[layout.scales + 12 * e: layout.scales + 12 * (e + 1)] = sc.view(np.uint8)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
