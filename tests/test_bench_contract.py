"""The bench's reference arm (CPU oracle) and its JSON line, on the CPU.

The reference arm times the oracle on a bounded sample of the block and must
print one JSON line with the same metric, unit, direction and config as the
GPU arm; under a multi-rank launch only rank 0 prints.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.strip()]


def test_reference_arm_line():
    sys.path.insert(0, ROOT)
    import bench
    lines = _run({"RANK": "0"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"] == bench.workload_config(1)
    # the per-step sample is named beside the workload it is drawn from
    assert d["sample_per_step"]["elements"] == 1024 * 4096
    assert d["sample_per_step"]["of_workload_elements"] == d["config"]["elements"]
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert 0.6 < d["size_ratio"] < 0.75


def test_reference_arm_other_ranks_are_silent():
    assert _run({"RANK": "1"}) == []


def test_clock_summary():
    # the bench line's `clocks`: median SM clock, highest max clock, every
    # throttle reason seen in the timed region, sample count and source
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.source = "test"
    c.samples = [(1965.0, 1965.0, set()), (1900.0, 1965.0, {"sw_power_cap"}), (1965.0, 1965.0, set()),
                 (1800.0, 1965.0, {"hw_slowdown"})]
    d = c.summary()
    assert d == {"sm_mhz": 1932.5, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown", "sw_power_cap"],
                 "samples": 4, "source": "test"}
    c.samples = []
    assert c.summary()["samples"] == 0 and c.summary()["sm_mhz"] is None
