"""The benchmark's reference arm (the fp64 oracle timed on the host cores)
prints one JSON line with the contract's keys; runs on CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--cpu-baseline-seconds", "0.3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["config"]["workload"] == "dense_p16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "2"], capture_output=True, text=True,
                       timeout=120, cwd=ROOT)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_reference_arm_under_a_launcher():
    """Launched with N ranks, rank 0 alone times the oracle and prints the
    line (naming N GPUs); every other rank exits 0 without work."""
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
            "--steps", "1", "--warmup", "3", "--cpu-baseline-seconds", "0.2"]
    other = subprocess.run(base, capture_output=True, text=True, timeout=120, cwd=ROOT,
                           env={**os.environ, "RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert other.returncode == 0 and other.stdout.strip() == ""
    first = subprocess.run(base, capture_output=True, text=True, timeout=300, cwd=ROOT,
                           env={**os.environ, "RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"})
    assert first.returncode == 0, first.stderr[-2000:]
    d = json.loads(first.stdout.strip())
    assert d["impl"] == "reference" and d["n_gpus"] == 2
