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
    assert line["config"]["workload"] == "opt125m-block"
    # six layers of 2048 tokens per step
    assert line["value"] == pytest.approx(
        6 * 2048 / (line["ms_per_step"] * 1e-3), rel=1e-6)
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0
    assert e2e["d2h_bytes_per_step"] > 0
    assert line["gpu_launches"] == 16 * steps
    if line["clocks"] is not None:
        assert line["clocks"]["sm_mhz"] > 0
