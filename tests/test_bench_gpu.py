"""The benchmark's JSON line on a B200: one short run of bench.py (without
the CPU baselines) in a child process, checked against the keys and
relations the line promises."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_keeps_its_contract():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS
    steps = 200
    r = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", str(steps),
         "--warmup", "3", "--no-cpu-baseline"], capture_output=True,
        text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == steps
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    wl = WORKLOADS["llama7b-prefill"]
    assert line["config"] == bench.workload_config(wl, 1)
    # three layers of 4096 tokens per step
    assert line["value"] == pytest.approx(
        3 * 4096 / (line["ms_per_step"] * 1e-3), rel=1e-6)
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    region = line["ms_per_step"] * steps / 1e3
    if roof["bound"] == "tensor":
        pk = bench.peaks()
        want = pk["bf16_tflops_sustained"] if region >= 1.0 else \
            pk["bf16_tflops"]
        assert roof["peak"] == want
    e2e = line["e2e"]
    assert e2e["value"] > 0
    # the three inputs in, the three outputs out, bf16
    assert e2e["h2d_bytes_per_step"] == 2 * 4096 * (4096 + 4096 + 11008)
    assert e2e["d2h_bytes_per_step"] == 2 * 4096 * (4096 + 11008 + 4096)
    # per input: statistics+scales and prepare; per layer: quantize, project
    assert line["gpu_launches"] == 12 * steps
    clocks = line["clocks"]
    assert clocks is not None and clocks["sm_mhz"] > 0
    assert clocks["in_timed_region"]
