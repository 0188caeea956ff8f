"""The reference arm's JSON line (CPU only, tiny shapes): the keys the bench
contract fixes, and a config identical to the native arm's when the whole
workload is timed."""
import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_line_matches_the_native_config(monkeypatch):
    shapes = (("qkv", 256, 128, 1), ("o_proj", 256, 64, 2), ("gate_up", 256, 256, 3), ("down", 512, 64, 4))
    monkeypatch.setattr(bench, "SHAPES", shapes)
    monkeypatch.setattr(bench, "STEP_BYTES", sum(bench.decode_bytes(1, K, N) for _, K, N, _ in shapes))
    monkeypatch.setattr(bench, "_ORACLE_W", {})
    line = bench.run_reference(argparse.Namespace(steps=2, warmup=3, gpus=1))
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["config"] == bench.workload_config(1)          # the whole workload: no sample key
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_workload_config_names_the_l2_rule_and_bytes():
    c = bench.workload_config(4)
    assert c["workload"] == bench.WORKLOAD and c["M"] == 1
    assert c["bytes_per_step"] == sum(bench.decode_bytes(1, K, N) for _, K, N, _ in bench.SHAPES)
    assert "L2" in c["l2"] and c["parallelism"] == "replicas x4"
