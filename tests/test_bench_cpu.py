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


def test_algorithmic_bytes_and_traffic_records():
    assert bench.algorithmic_bytes(8192, 14336) == 297271296.0
    for row, kern in bench.TRAFFIC_KERNEL.items():
        assert row in bench.CONFIG_ROWS and kern in bench.KERNEL_SOURCES
        path = os.path.join(ROOT, "profiles", f"traffic_{row}.json")
        if not os.path.exists(path):
            assert bench.recorded_traffic(row) is None
            continue
        rec = json.load(open(path))
        assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
        # the recorded traffic is reported only while the kernel source is unchanged
        t = bench.recorded_traffic(row)
        assert t is None or abs(t - rec["dram_bytes_per_launch"]) < 1


def test_rotating_sets_exceed_l2():
    for set_bytes in (85e6, 297e6, 1.19e9, 1.36e9):
        n = bench._sets_for(set_bytes)
        assert n >= 2 and n * set_bytes >= 3 * bench.L2_BYTES


def test_peak_source():
    peak, kind = bench.hbm_peak()
    assert peak > 1000 and kind in ("measured", "fallback")
