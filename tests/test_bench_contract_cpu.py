"""bench.py's reference arm (the fp64 oracle on the host cores) at N = 1, run in-process on
the CPU: one JSON line with every key of the benchmark contract, on the same metric, unit
and workload as the GPU arm."""
import io
import json
import os
from contextlib import redirect_stdout

import bench

CONTRACT_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                 "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_line_at_one_rank(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert rc == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1, lines
    line = json.loads(lines[0])
    assert CONTRACT_KEYS <= set(line), CONTRACT_KEYS - set(line)
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"] == "causal_mha_b8_h32_n4096_d128"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_recorded_traffic_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    # a traffic figure is only reported while the measured sources are unchanged
    import hashlib

    from io_aware_softmax_b200 import build as b
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    (csrc / "k.cu").write_text("__global__ void k() {}\n")
    digest = hashlib.sha256((csrc / "k.cu").read_bytes()).hexdigest()
    root = tmp_path / "root"
    (root / "profiles").mkdir(parents=True)
    (root / "profiles" / "traffic.json").write_text(json.dumps(
        {"kern": {"bytes_per_launch": 1234, "sources": ["k.cu"], "sha256": digest}}))
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setattr(b, "CSRC", str(csrc))
    assert bench.recorded_traffic("kern") == 1234
    assert bench.recorded_traffic("other") is None
    (csrc / "k.cu").write_text("__global__ void k() { /* changed */ }\n")
    assert bench.recorded_traffic("kern") is None
    assert os.path.exists(root / "profiles" / "traffic.json")

