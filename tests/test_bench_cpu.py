"""The benchmark's reference arm (the CPU oracle on the host cores) and its
JSON line, on the small workload; no GPU needed."""
import os
import types

import bench


def test_reference_arm_line(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    out = bench.run_reference(types.SimpleNamespace(workload="tiny", steps=2, warmup=1))
    assert out["impl"] == "reference" and out["unit"] == "TFLOP/s" and out["value"] > 0
    assert out["higher_is_better"] is True and out["steps"] == 2 and out["warmup"] == 1
    assert out["config"]["workload"].startswith("tiny ")
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == out["value"] and cb["cores"] == len(os.sched_getaffinity(0))
    assert out["e2e"] == {"value": out["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_only_on_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(types.SimpleNamespace(workload="tiny", steps=1, warmup=0)) is None
