"""Host-side checks of the C ABI (CPU only: nothing here launches a kernel).

The shared library must load and export every entry point that
include/moe_b200.h declares, and its size / layout queries and argument
validation must behave as the header states.
"""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from fp8_moe_expert_top_b200 import binding as B

from helpers import sf_index

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(B.LIB_PATH):
        from fp8_moe_expert_top_b200 import build
        build.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 14
    L = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    # and the binding covers every one of them
    assert set(names) == set(B.SIGNATURES), set(names) ^ set(B.SIGNATURES)


def test_config_validation():
    ok = B.make_config(384, 8, 4096, 2560, "nvfp4")
    assert B.moe_check_config(ok) == 0
    assert B.moe_check_config(B.make_config(8, 2, 256, 128, "mxfp8")) == 0
    for bad in [B.make_config(384, 9, 4096, 2560, 0), B.make_config(384, 8, 4000, 2560, 0),
                B.make_config(384, 8, 4096, 2500, 0), B.make_config(0, 1, 256, 128, 0),
                B.make_config(2048, 8, 256, 128, 0), B.make_config(4, 8, 256, 128, 0),
                B.make_config(8, 2, 256, 128, 7)]:
        assert B.moe_check_config(bad) == 2


def test_max_rows_bound():
    cfg = B.make_config(384, 8, 4096, 2560, "nvfp4")
    for T in [0, 1, 7, 64, 8192, 16384]:
        R = B.moe_max_rows(cfg, T)
        slots = T * 8
        assert R % 128 == 0
        assert R >= slots + 127 * min(384, slots) - 127
        # the worst case (every touched expert one slot past a multiple of 128) fits
        assert R >= sum(((c + 127) // 128) * 128 for c in [1] * min(384, slots) + [0]) if slots else R == 0
    assert B.moe_max_rows(cfg, -1) == -1


def test_sf_offset_matches_layout_contract():
    rows, nsf = 256, 16
    idx = sf_index(rows, nsf)
    for r in [0, 1, 31, 32, 63, 127, 128, 200, 255]:
        for c in [0, 1, 3, 4, 7, 15]:
            assert B.moe_sf_offset(r, c, nsf) == idx[r, c]
    # the map is a bijection onto [0, rows * nsf)
    assert np.array_equal(np.sort(idx.reshape(-1)), np.arange(rows * nsf))


def test_sizes():
    cfg = B.make_config(384, 8, 4096, 2560, "nvfp4")
    assert B.moe_codes_bytes(cfg, 128, 4096) == 128 * 2048
    assert B.moe_sf_bytes(cfg, 128, 4096) == 128 * 256
    assert B.moe_sf_bytes(cfg, 100, 4096) == -1
    cfg8 = B.make_config(384, 8, 4096, 2560, "mxfp8")
    assert B.moe_codes_bytes(cfg8, 128, 4096) == 128 * 4096
    assert B.moe_sf_bytes(cfg8, 128, 4096) == 128 * 128
    L = B.moe_get_weights_layout(cfg)
    E, H, I = 384, 4096, 2560
    assert L.w13_sf - L.w13_codes >= E * 2 * I * H // 2
    assert L.w2_codes - L.w13_sf >= E * 2 * I * H // 16
    assert L.total_bytes >= L.scales + E * 12
    for off in (L.w13_codes, L.w13_sf, L.w2_codes, L.w2_sf, L.scales):
        assert off % 256 == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers: run only where nothing can launch")
def test_invalid_arguments_are_rejected_before_any_launch():
    """Null or misaligned pointers and small workspaces return a status, with no
    CUDA call made (these run on a machine without a GPU)."""
    cfg = B.make_config(8, 2, 256, 128, "nvfp4")
    L = B.lib()
    null = None
    st = L.moe_route_topk(ctypes.byref(cfg), 4, null, null, null, null, null, null, null, null, 0, null)
    assert st == 1
    fake = ctypes.c_void_p(0x10000)
    st = L.moe_route_topk(ctypes.byref(cfg), 4, fake, fake, fake, fake, fake, fake, fake, fake, 1, null)
    assert st == 3           # workspace too small
    mis = ctypes.c_void_p(0x10004)
    st = L.moe_permute(ctypes.byref(cfg), 4, mis, fake, fake, fake, fake, null)
    assert st == 1           # misaligned x
    st = L.moe_permute(ctypes.byref(cfg), 4, fake, null, fake, fake, fake, null)
    assert st == 1           # NVFP4 needs the activation scale
    st = L.moe_forward(ctypes.byref(cfg), 4, null, fake, fake, fake, fake, fake, fake, fake, fake, fake, null, null,
                       null)
    assert st == 1
    bad = B.make_config(8, 2, 250, 128, "nvfp4")
    st = L.moe_unpermute_combine(ctypes.byref(bad), 4, fake, fake, fake, fake, null)
    assert st == 2
    st = L.moe_quantize_weights(ctypes.byref(cfg), 6, 4, fake, fake, fake, fake, null)
    assert st == 1           # expert range past E
    # T == 0 is a valid no-op for the calls that need no pointers
    assert L.moe_permute(ctypes.byref(cfg), 0, null, null, null, null, null, null) == 0
    assert B.lib().moe_status_string(3) == b"workspace too small"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    mod = importlib.import_module("fp8_moe_expert_top_b200.binding")
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()
