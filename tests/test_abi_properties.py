"""Properties of the C ABI's size and layout queries (CPU only, no kernel).

  * moe_max_rows(T) bounds the rows that any routing of T tokens can occupy:
    the oracle's slot sort (128-padded expert segments) of random and of
    adversarial routings never needs more, and the adversarial case (every
    touched expert one slot past a multiple of 128) reaches the bound.
  * moe_sf_offset is a bijection from (row, scale column) onto the bytes of a
    scale buffer of moe_sf_bytes, whole 512-byte atoms of 128 rows x 4 columns.
  * moe_route_workspace_bytes and moe_codes_bytes grow monotonically.
"""

import numpy as np
from hypothesis import example, given, settings, strategies as st

from fp8_moe_expert_top_b200 import binding as B
from oracle import route as rt


def _cfg(E, k):
    return B.make_config(E, k, 256, 128, "nvfp4")


def _random_ids(rng, T, E, k, skew):
    """T tokens, each with k distinct experts; `skew` concentrates them."""
    p = np.exp(-skew * np.arange(E) / max(E - 1, 1))
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]) if T else np.zeros((0, k), int)


@settings(max_examples=60, deadline=None, derandomize=True)
@given(E=st.integers(8, 512), k=st.integers(1, 8), T=st.integers(0, 1500), skew=st.floats(0.0, 8.0),
       seed=st.integers(0, 2 ** 31 - 1))
def test_max_rows_bounds_every_routing(E, k, T, skew, seed):
    cfg = _cfg(E, k)
    assert B.moe_check_config(cfg) == 0
    ids = _random_ids(np.random.default_rng(seed), T, E, k, skew)
    _, offsets, sorted_slots, _ = rt.sort_slots(ids, E)
    R = B.moe_max_rows(cfg, T)
    assert R % 128 == 0
    assert offsets[-1] <= R
    assert sorted_slots.shape[0] == offsets[-1]


@settings(max_examples=40, deadline=None, derandomize=True)
@given(E=st.integers(8, 512), k=st.integers(1, 8), m=st.integers(1, 64))
@example(E=8, k=2, m=8)           # every expert touched: the bound is reached
@example(E=48, k=8, m=48)
def test_max_rows_reached_by_adversarial_routing(E, k, m):
    """m experts (m <= E) each get 128 q + 1 slots; when they can take every
    slot of T tokens the padded rows reach moe_max_rows exactly."""
    m = min(m, E)
    if m < k:
        return
    counts = np.full(m, 129)                  # one past a multiple of 128
    S = int(counts.sum())
    if S % k:
        return
    T = S // k
    # deal slots round-robin so each token's k experts are distinct (m >= k)
    order = np.arange(S) % m
    ids = order.reshape(T, k)
    assert all(len(set(row)) == k for row in ids.tolist())
    _, offsets, _, _ = rt.sort_slots(ids, E)
    assert offsets[-1] == m * 256
    R = B.moe_max_rows(_cfg(E, k), T)
    assert offsets[-1] <= R
    if m == min(E, S):                          # every possible expert touched: the bound is tight
        assert R == offsets[-1]


@settings(max_examples=25, deadline=None, derandomize=True)
@given(blocks=st.integers(1, 3), atoms=st.integers(1, 6))
def test_sf_offset_is_a_bijection_onto_the_scale_buffer(blocks, atoms):
    rows, nsf = 128 * blocks, 4 * atoms
    L = B.lib()
    offs = np.array([[L.moe_sf_offset(r, c, nsf) for c in range(nsf)] for r in range(rows)], dtype=np.int64)
    cfg = B.make_config(8, 2, 256, 128, "nvfp4")            # a valid config; K = 16 * nsf for NVFP4
    assert B.moe_sf_bytes(cfg, rows, 16 * nsf) == rows * nsf
    assert np.array_equal(np.sort(offs.reshape(-1)), np.arange(rows * nsf))
    # one atom = 128 consecutive rows x 4 consecutive columns, 512 bytes
    for r0 in range(0, rows, 128):
        for c0 in range(0, nsf, 4):
            a = offs[r0:r0 + 128, c0:c0 + 4]
            assert a.min() % 512 == 0 and a.max() - a.min() == 511


def test_size_queries_grow_with_the_batch():
    cfg = B.make_config(384, 8, 4096, 2560, "nvfp4")
    Ts = [0, 1, 2, 3, 16, 17, 64, 100, 1000, 8192, 8193, 40000]
    ws = [B.moe_route_workspace_bytes(cfg, T) for T in Ts]
    rows = [B.moe_max_rows(cfg, T) for T in Ts]
    assert all(a <= b for a, b in zip(ws, ws[1:]))
    assert all(a <= b for a, b in zip(rows, rows[1:]))
    codes = [B.moe_codes_bytes(cfg, r, 4096) for r in rows[1:]]
    assert all(a <= b for a, b in zip(codes, codes[1:]))
