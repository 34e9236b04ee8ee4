"""The JSON line of bench.py's reference arm (the float64 oracle timed on the
host cores), checked on CPU: rank 0 of a one-process job prints exactly one
line with every key the benchmark contract asks for."""
import contextlib
import io
import json
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_reference_arm_line_has_the_contract_keys(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("LOCAL_RANK", "0")
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    # the arm's default workload is the 720p-like training step ...
    assert bench.workload_of(args).N == 76800 and bench.workload_of(args).heads == 40
    # ... whose oracle sample takes ~20 s of CPU; the line's keys are checked
    # on the small workload's sample instead
    from adaptive_block_sparse_fractal_b200 import synth
    monkeypatch.setattr(bench, "workload_of", lambda a: synth.WORKLOADS["small"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args) == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])

    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 1, 3)
    assert line["ms_per_step"] > 0
    assert line["higher_is_better"] is True
    assert line["scaling"] == "strong"
    assert line["vs_baseline"] is None
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    # the same workload as the CUDA arm's line
    assert line["config"] == bench.workload_config(bench.workload_of(args))
    assert line["ms_per_step_kind"] == "extrapolated from a timed sample"

    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["unit"] == "TFLOP/s"
    assert cb["value"] == pytest.approx(line["value"])
    assert cb["cores"] >= 1 and "8 sampled query blocks" in cb["sample"]
    assert "backward" in cb["sample"] and "extrapolated" in cb["sample"]
    # the line's time is the extrapolated whole step, consistent with its value
    assert cb["extrapolated_ms_per_step"] == pytest.approx(line["ms_per_step"])

    e2e = line["e2e"]
    assert e2e["value"] == pytest.approx(line["value"]) and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.main()
