"""bench.py's reference arm (the oracle on the host cores) needs no GPU: run it
on the small workload and check its JSON line field by field."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _reference_line(*extra):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_l2k",
                        "--steps", "2", "--warmup", "1", *extra],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    j = _reference_line()
    assert j["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["n_gpus"] == 1 and j["steps"] == 2 and j["warmup"] == 1
    assert j["higher_is_better"] is True and j["vs_baseline"] is None
    assert j["value"] > 0 and j["ms_per_step"] > 0
    assert j["config"]["workload"] == "tiny_l2k"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["unit"] == j["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_fp8_indexer_line():
    j = _reference_line("--fp8")
    assert j["config"]["fp8_indexer"] is True and j["value"] > 0


def test_reference_arm_declines_the_sweep_and_unknown_workloads():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "hier_sweep"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    j = json.loads(r.stdout.strip().splitlines()[-1])
    assert j["impl"] == "reference" and "hier_sweep" in j["unavailable"]
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "no_such_workload"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "invalid choice" in r.stderr
