"""bench.py on the GPU, on a small slice of the KAT-B workload: one JSON line
with the keys and units the measurement contract asks for, a roofline and an
ALU roofline for the backward kernel, tensor rooflines for the fused linear
layer, the end-to-end leg through host buffers, the determinism check, and
per-workload timings."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--rows", "4000", "--steps", "5",
           "--warmup", "3", "--no-cpu-baseline", "--e2e-steps", "2", "--fused-launches", "3",
           "--linear-nout", "512", "--per-config", "kat_t,stress:64", "--per-config-steps", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "roofline_alu", "e2e", "gpu_launches", "clocks", "determinism"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["dtype"] == "f32"
    assert d["config"]["workload"] == "kat_b" and d["config"]["dtype"] == "bf16"
    assert d["config"]["kernel_path"] == {"forward": "tma", "backward": "tma"}
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] < 1.5
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["roofline_alu"]["bound"] == "alu"
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] == 2 * 4000 * 3072 * 2
    assert d["gpu_launches"] == 5 * 3
    assert d["determinism"]["dA_dB_identical_over_steps"] is True
    assert d["clocks"] is None or d["clocks"]["samples"] >= 1
    assert [c["workload"] for c in d["per_config"]] == ["kat_t", "stress_ng64"]
    fl = d["fused_linear"]
    assert fl["nout"] == 512 and fl["kernel"] == "one CTA per tile"
    for part in (fl, fl["backward"]):
        r = part["roofline"]
        assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and 0 < r["frac"] < 1.5
        assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
        assert r["flops_per_launch"] == 2.0 * 4000 * 3072 * 512
    assert d["device_error"] == 0
