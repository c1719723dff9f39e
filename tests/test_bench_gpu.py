"""bench.py's JSON line on the GPU, for each of its modes, on small inputs:
the contract's keys are there, the numbers are sane, and the dominant
kernel's roofline fraction is a fraction of the measured peak."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"}

MODES = {
    "default": ["--psi", "8388608", "--steps", "20", "--warmup", "3"],
    "eager": ["--psi", "8388608", "--steps", "20", "--warmup", "3", "--eager", "--no-cpu-baseline"],
    "stage3_prefetch": ["--config", "stage3_1p3b", "--layers", "2", "--steps", "2", "--warmup", "3",
                        "--prefetch", "1", "--no-cpu-baseline", "--no-e2e"],
    "guarded": ["--guarded", "--psi", "8388608", "--steps", "5", "--warmup", "3"],
    "peer": ["--peer", "--psi", "8388608", "--steps", "5", "--warmup", "3"],
    "reshard": ["--reshard", "6", "--psi", "8388608", "--steps", "5", "--warmup", "3"],
    "adamw": ["--weight-decay", "0.01", "--psi", "8388608", "--steps", "5", "--warmup", "3",
              "--no-cpu-baseline", "--no-e2e"],
}


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("mode", sorted(MODES))
def test_bench_line(mode):
    r = subprocess.run([sys.executable, "bench.py"] + MODES[mode], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert KEYS <= set(line), KEYS - set(line)
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["n_gpus"] == 1
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert 0.05 < roof["frac"] < 1.3, roof
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    assert line["gpu_launches"] > 0
    assert line["clocks"] is None or "sm_mhz" in line["clocks"]
    if mode in ("default", "eager"):
        # the kernel is timed in the timed steps: its launches fit in the step
        assert roof["avg_launch_ms"] * line["config"]["buckets"] <= line["ms_per_step"] * 1.001
        assert "timing" in roof and roof["isolated"]["frac"] > 0
        assert abs(roof["frac_of_nominal"] * roof["nominal_peak"] - roof["achieved"]) < 1e-6
    if mode == "default":
        assert line["config"]["graph"] is True
        assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["value"] > 0
        assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] > 0
        allc = line["cpu_baseline_all_cores"]
        assert allc["cores"] >= 1 and allc["value"] > 0
    if mode == "eager":
        assert line["config"]["graph"] is False
    if mode == "stage3_prefetch":
        assert line["config"]["prefetch"] == 1 and line["config"]["peak_live_units"] == 2
    if mode == "adamw":
        assert line["config"]["weight_decay"] == 0.01
