"""The benchmark's contract pieces that run without a GPU.

  * The reference arm times the CPU oracle on a bounded sample of the decode
    step and prints one JSON line with the keys the harness reads; ranks
    other than 0 print nothing.
  * The roofline's DRAM traffic comes from the committed record of the ncu
    capture of the decode kernel and is reported only while the record's
    hash of the kernel's device sources is the current one.
"""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CMD = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"]


def _json_lines(stdout):
    return [json.loads(line) for line in stdout.splitlines() if line.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run(CMD, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["config"]["workload"] == bench.WORKLOAD
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"] == line["config"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run(CMD, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert _json_lines(r.stdout) == []


def test_traffic_is_reported_only_for_the_profiled_source(monkeypatch):
    rec = json.load(open(bench.TRAFFIC_FILE))
    assert rec["sources"] == list(bench.DECODE_SOURCES)
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    monkeypatch.setattr(bench, "decode_source_hash", lambda: rec["sources_sha256_16"])
    assert bench.committed_traffic() == float(rec["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "decode_source_hash", lambda: "0" * 16)
    assert bench.committed_traffic() is None

