"""The bench's JSON line (one short run of the decode workload): every key
the line promises, with consistent values."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _recorded_traffic():
    """The DRAM bytes per 30-layer launch that bench.py records from its ncu
    capture (read from its source, so the test follows a new capture)."""
    import ast
    with open(os.path.join(ROOT, "bench.py")) as f:
        tree = ast.parse(f.read())
    for node in tree.body:
        if isinstance(node, ast.Assign) and any(
                isinstance(t, ast.Name) and t.id == "NCU_TRAFFIC" for t in node.targets):
            return ast.literal_eval(node.value)["moe_decode_kernel"]["bytes"]
    raise AssertionError("bench.py records no NCU_TRAFFIC")


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
    if rf["traffic"] is not None:   # the recorded 30-layer traffic, scaled to 2 layers
        assert rf["traffic"] == round(_recorded_traffic() * 2 / 30)
    e2e = d["e2e"]
    assert e2e["unit"] == "layers/s" and e2e["h2d_bytes_per_step"] == 2 * 2816 * 2
    assert e2e["d2h_bytes_per_step"] == 2 * 2816 * 2
    assert d["gpu_launches"] == 20
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
