"""The reference arm of bench.py (the CPU oracle timed on the headline
workload): the JSON line it prints on rank 0, and that other ranks do no work."""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _run(monkeypatch, capsys, rank: int, world: int):
    monkeypatch.setenv("RANK", str(rank))
    monkeypatch.setenv("WORLD_SIZE", str(world))
    monkeypatch.setenv("LOCAL_RANK", str(rank))
    bench.run_reference(argparse.Namespace(steps=1, warmup=3))
    return capsys.readouterr().out.strip().splitlines()


def test_reference_line_matches_our_arm(monkeypatch, capsys):
    lines = _run(monkeypatch, capsys, 0, 1)
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    # the same metric, unit, direction, workload and inputs as our arm's line
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["config"]["workload"] == bench.WORKLOAD and line["data"] == bench.DATA
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1
    assert cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_other_ranks_exit_without_work(monkeypatch, capsys):
    assert _run(monkeypatch, capsys, 1, 2) == []
