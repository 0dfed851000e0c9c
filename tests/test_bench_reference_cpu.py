"""The benchmark's reference arm runs on the host alone: with no reference
implementation to install, `bench.py --impl reference` times the fp64 oracle
on the host cores and prints one JSON line in the bench contract's format."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["S"] == 75600 and d["config"]["H"] == 40


def test_clock_summary_keeps_the_samples_of_the_timed_region(tmp_path):
    """The bench's clock record: timestamped nvidia-smi lines, of which only
    those between the marks of the timed region count (median SM clock, the
    highest max clock, every throttle reason seen active)."""
    import datetime
    import time
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.proc = object()                                   # stands for the sampler process
    path = tmp_path / "clocks.csv"
    now = time.time()
    lines = []
    for i, dt in enumerate([-2.0, -0.5, 0.1, 0.3, 0.5, 2.0]):
        ts = datetime.datetime.fromtimestamp(now + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        cap = "Active" if i == 3 else "Not Active"
        slow = "Active" if i == 0 else "Not Active"        # outside the region: must not count
        lines.append(f"{ts}, 0, {1500 + 10 * i}, 1965, 700.0, 0x4, {slow}, Not Active, Not Active, {cap}")
    path.write_text("\n".join(lines) + "\n")
    c.file = open(path)
    c.t0, c.t1 = now, now + 0.6
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1530.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
