"""The bench's JSON contract, checked on the host: the reference arm (the
fp64 oracle timed on the CPU) prints exactly one JSON line with the keys the
benchmark contract names, for a small workload; under a non-zero RANK it
prints nothing."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(args, env=None):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                       timeout=300, env=dict(os.environ, **(env or {})), cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [l for l in r.stdout.splitlines() if l.strip()]


def test_reference_arm_prints_one_contract_line():
    lines = run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("tiny")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_is_silent_on_other_ranks():
    assert run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "1"],
               env={"RANK": "1", "WORLD_SIZE": "2"}) == []


FAKE_SMI = """#!/bin/sh
# stands in for nvidia-smi's CSV query loop: index, SM MHz, max SM MHz,
# power W, then the five clock-event reason columns
while true; do
  echo "0, 1800, 1965, 650.5, 0x4, Not Active, Not Active, Not Active, Active"
  echo "0, 1700, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active"
  sleep 0.05
done
"""


def test_clock_sampler_reads_the_query_loop(tmp_path, monkeypatch):
    """The sampler runs the query loop during the timed region and reduces
    it to the median SM clock under load (samples above 300 W), the maximum
    clock and the active reasons; here against a stand-in nvidia-smi."""
    import time
    sys.path.insert(0, ROOT)
    import bench
    smi = tmp_path / "nvidia-smi"
    smi.write_text(FAKE_SMI)
    smi.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    with bench.ClockSampler(0) as clk:
        time.sleep(0.4)
    s = clk.summary()
    assert s["samples"] >= 2 and s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 650.5
    assert clk.proc.poll() is not None                 # the loop was stopped
