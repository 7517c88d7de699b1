"""bench.py's contract pieces that run without a GPU: the reference arm's JSON line
(the CPU oracle on a bounded sample of the bench workload) and the roofline helpers."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["rows"] == 8192 and line["config"]["cols"] == 14336


def test_algorithmic_bytes_and_traffic_record():
    assert bench.algorithmic_bytes(8192, 14336) == 297271296.0
    rec = json.load(open(bench.TRAFFIC_FILE))
    assert rec["algorithmic_bytes_per_launch"] == 297271296.0
    # the recorded traffic is reported only while the kernel source is unchanged
    t = bench.recorded_traffic()
    assert t is None or abs(t - rec["dram_bytes_per_launch"]) < 1


def test_peak_source():
    peak, kind = bench.hbm_peak()
    assert peak > 1000 and kind in ("measured", "fallback")
