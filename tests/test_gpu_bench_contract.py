"""The bench's JSON line (one short run of the decode workload): every key
the line promises, with consistent values."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.slow
def test_decode_bench_line(cuda_dev):
    out = subprocess.run([sys.executable, "bench.py", "--layers", "2", "--steps", "20",
                          "--warmup", "3", "--no-cpu-baseline"], cwd=ROOT, capture_output=True,
                         text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3
    assert d["unit"] == "layers/s" and d["higher_is_better"] is True
    assert d["value"] == pytest.approx(2 * 1e3 / d["ms_per_step"], rel=1e-3)
    assert "workload" in d["config"] and d["config"]["layers"] == 2
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and rf["peak"] > 0
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], rel=1e-3)
    if rf["traffic"] is not None:   # the 30-layer capture, scaled to 2 layers
        assert rf["traffic"] == pytest.approx(933512960 * 2 / 30, rel=1e-6)
    e2e = d["e2e"]
    assert e2e["unit"] == "layers/s" and e2e["h2d_bytes_per_step"] == 2 * 2816 * 2
    assert e2e["d2h_bytes_per_step"] == 2 * 2816 * 2
    assert d["gpu_launches"] == 20
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
