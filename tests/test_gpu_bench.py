"""bench.py's GPU arm on a reduced problem (2 of the 720p-like shape's 40
heads): the JSON line carries the contract's keys, the roofline and clock
records, and the end-to-end step -- run in (batch, head) chunks on two copy
streams -- gives the device-resident step's outputs bit for bit."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

pytestmark = pytest.mark.gpu


def test_bench_line_two_heads(capsys):
    args = bench.parse(["--heads", "2", "--steps", "2", "--warmup", "3", "--no-sweep", "--no-cpu"])
    assert bench.run_nabla(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "clocks", "gpu_launches", "breakdown_ms"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["value"] > 0
    assert line["gpu_launches"] == 11 * 2
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"])
    e2e = line["e2e"]
    assert e2e["outputs_match_device_step"] is True
    assert e2e["h2d_bytes_per_step"] == 4 * 2 * 76800 * 128 * 2
    assert e2e["d2h_bytes_per_step"] == 4 * 2 * 76800 * 128 * 2
    assert e2e["ms_per_step"] >= line["ms_per_step"] * 0.5
