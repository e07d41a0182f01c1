"""The benchmark's command-line contract, on CPU.

The reference arm (`--impl reference`) times the oracle on the host, so its
JSON line can be checked here: the keys and their types, the workload name,
and, under torchrun with two ranks (gloo, CPU), that rank 0 alone prints one
line and every rank exits 0.  The GPU arm needs a B200 and must fail loudly
without one (no JSON line, non-zero exit) rather than fall back to the CPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REF_ARGS = ["--impl", "reference", "--workload", "tiny_nvfp4", "--steps", "3", "--warmup", "3"]


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def _check_reference_line(d):
    for key, typ in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                     ("dtype", str), ("data", str), ("config", dict), ("cpu_baseline", dict), ("e2e", dict)):
        assert isinstance(d[key], typ), (key, d.get(key))
    assert d["impl"] == "reference"
    assert d["vs_baseline"] is None
    assert d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_nvfp4"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", *REF_ARGS], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_two_ranks():
    for _ in range(3):            # the free port can be taken between the probe and torchrun's bind
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
               "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
               *REF_ARGS]
        r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
        if r.returncode == 0 or "address already in use" not in r.stderr.lower():
            break
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0])


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_gpu_arm_fails_loudly_without_gpu():
    r = subprocess.run([sys.executable, "bench.py", "--steps", "3", "--warmup", "3"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert _json_lines(r.stdout) == []


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_match_the_published_sizes():
    """The roofline's numerators: packed weights of all 384 experts are 6.795
    GB (NVFP4, 0.5625 B per element) and 12.457 GB (MXFP8, 1.03125 B) per
    layer, 31,457,280 elements per expert; the layer's other compulsory bytes
    are x and y in bf16 and the float32 logits."""
    bench = _bench_module()
    from fp8_moe_expert_top_b200 import inputs
    for name, per_layer in (("prefill_nvfp4", 6.795e9), ("prefill_mxfp8", 12.457e9)):
        wl = inputs.WORKLOADS[name]
        H, I, E, T = wl.d_model, wl.d_ffn, wl.num_experts, wl.T
        assert 3 * H * I == 31_457_280
        b = bench.phase_bytes(wl, E, T * wl.top_k)
        weights = b["layer"] - (T * H * 2 + T * E * 4 + T * H * 2)
        assert abs(weights - per_layer) <= 0.0005 * per_layer, (name, weights)
        assert b["gateup"] - (2 * weights / 3) == pytest.approx(T * wl.top_k * (H + I) * (weights / E / (3 * H * I)))
        # every phase's bytes are positive and the layer excludes the permuted buffers
        assert all(v > 0 for v in b.values())
        assert b["layer"] < sum(b[p] for p in bench.PHASES)

