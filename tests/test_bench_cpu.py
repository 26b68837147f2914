"""bench.py on the CPU: the reference arm (the oracle, timed on host cores) prints one
JSON line with the contract's keys; the recorded-traffic lookup follows the sweep
sources."""
import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(__file__), "..")


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "c1",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.strip().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"].startswith("c1 ")
    # the oracle runs on every core of the host, and says so
    cores = len(os.sched_getaffinity(0))
    assert d["cpu_baseline"]["cores"] == cores
    assert d["cpu_baseline"]["cpu_model"] and d["cpu_baseline"]["extrapolated"] is False


def test_recorded_traffic_is_tied_to_the_sweep_sources():
    sys.path.insert(0, ROOT)
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    h = bench.kernel_source_hash()
    for key in ("fp16x3/tc_lse", "fp16x3/tc_stats"):
        got = bench.recorded_traffic(key.split("/")[1], "fp16x3")
        if rec[key]["source_hash"] == h:
            assert got == rec[key]["bytes_per_launch"] and got > 0
        else:
            assert got is None
    assert bench.recorded_traffic("tc_lse", "fp32") is None
