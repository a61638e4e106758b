"""bench.py's reference arm (the CPU oracle timed on a bounded sample) prints
one JSON line with the contract's keys; runs on the CPU in a few seconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_traffic_table_entries_are_well_formed():
    """Every DRAM-traffic entry names existing library sources, a hash of them,
    a positive byte count and a note; a stale entry (sources changed since the
    capture) is reported as null with its reason, never as a number."""
    sys.path.insert(0, ROOT)
    import bench
    for key, e in bench.NCU_TRAFFIC.items():
        assert len(key) == 4 and key[3] in ("decode", "cascade", "prefill"), key
        assert e["bytes"] > 0 and e["note"], key
        for f in e["files"]:
            assert os.path.exists(os.path.join(bench.CSRC, f)), (key, f)
        value, why = bench.ncu_traffic(key)
        if bench.src_hash(e["files"]) == e["sha"]:
            assert value == e["bytes"], key
        else:
            assert value is None and why.startswith("stale"), key
    assert bench.ncu_traffic(("no such workload", "bfloat16", 0, "decode")) == (None, "no capture of this configuration")
