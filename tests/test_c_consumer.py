"""The C ABI from plain C (CPU only: nothing here launches a kernel).

tests/c_consumer.c includes include/moe_b200.h as strict C11 and links
libmoe_b200.so with no C++ and no torch; its host-side results must equal the
Python binding's.  The header must also compile as C++ (its extern "C" guard).
"""

import os
import shutil
import subprocess

import pytest

from fp8_moe_expert_top_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
SOURCE = os.path.join(ROOT, "tests", "c_consumer.c")


@pytest.fixture(scope="module")
def library():
    if not os.path.exists(B.LIB_PATH):
        from fp8_moe_expert_top_b200 import build
        build.build()
    return B.LIB_PATH


@pytest.fixture(scope="module")
def c_output(library, tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    out_dir = tmp_path_factory.mktemp("c_consumer")
    exe = str(out_dir / "c_consumer")
    lib_dir = os.path.dirname(library)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, SOURCE, "-o", exe,
                    "-L", lib_dir, "-lmoe_b200", f"-Wl,-rpath,{lib_dir}"], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    lines = {}
    for line in r.stdout.splitlines():
        key, *vals = line.split(" ", 1)
        lines.setdefault(key, []).append(vals[0] if vals else "")
    return lines


def _ints(s):
    return [int(v) for v in s.split()]


def test_config_checks(c_output):
    assert _ints(c_output["check"][0]) == [0, 0, 2]


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_weights_layout_matches_binding(c_output, fmt):
    st, *offs = _ints(c_output[f"layout_{fmt}"][0])
    assert st == 0
    lay = B.moe_get_weights_layout(B.make_config(384, 8, 4096, 2560, fmt))
    assert offs == [lay.w13_codes, lay.w13_sf, lay.w2_codes, lay.w2_sf, lay.scales, lay.total_bytes]


def test_row_and_workspace_queries_match_binding(c_output):
    cfg = B.make_config(384, 8, 4096, 2560, "nvfp4")
    rows = [_ints(s) for s in c_output["rows"]]
    assert [r[0] for r in rows] == [0, 1, 8, 64, 512, 4096]
    for T, r_max, ws in rows:
        assert r_max == B.moe_max_rows(cfg, T)
        assert ws == B.moe_route_workspace_bytes(cfg, T)


def test_buffer_sizes_and_scale_offsets_match_binding(c_output):
    nv = B.make_config(384, 8, 4096, 2560, "nvfp4")
    mx = B.make_config(384, 8, 4096, 2560, "mxfp8")
    assert _ints(c_output["codes"][0]) == [B.moe_codes_bytes(nv, 128, 4096), B.moe_codes_bytes(mx, 128, 4096),
                                          B.moe_sf_bytes(nv, 128, 4096), B.moe_sf_bytes(mx, 256, 2560)]
    L = B.lib()
    assert _ints(c_output["sf_offset"][0]) == [L.moe_sf_offset(130, 5, 256), L.moe_sf_offset(31, 3, 4)]


def test_status_codes_from_c(c_output):
    assert c_output["status_string"][0] == "workspace too small"
    assert _ints(c_output["null_logits"][0]) == [1]       # MOE_ERR_INVALID_ARG
    assert _ints(c_output["bad_config"][0]) == [2]        # MOE_ERR_UNSUPPORTED
    assert _ints(c_output["empty_permute"][0]) == [0]     # T = 0 is a no-op


def test_header_compiles_as_cxx(tmp_path):
    if shutil.which("g++") is None:
        pytest.skip("g++ not found")
    src = tmp_path / "h.cpp"
    src.write_text('#include "moe_b200.h"\n'
                   'static_assert(sizeof(moe_config) == 20, "moe_config is five int32");\n'
                   'static_assert(sizeof(moe_weights_layout) == 48, "moe_weights_layout is six int64");\n'
                   'int main() { moe_config c{384, 8, 4096, 2560, MOE_NVFP4}; return moe_check_config(&c); }\n')
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-I", INCLUDE,
                    str(src)], check=True, capture_output=True, text=True)
