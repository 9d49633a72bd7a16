"""The reference arm of bench.py keeps the JSON-line contract on the CPU (the oracle timed on
the host's cores for one decode query at 1M context), and ranks other than 0 exit quietly."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, env_extra=None, timeout=600):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=timeout)
    return r.returncode, r.stdout, r.stderr


def test_reference_arm_line():
    rc, out, err = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert rc == 0, err[-2000:]
    lines = [l for l in out.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "queries/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["config"]["workload"] == "decode_b1_1m"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "sample" in cb
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    rc, out, err = run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                             env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2",
                                        "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": "29531"}, timeout=120)
    assert rc == 0, err[-2000:]
    assert not [l for l in out.splitlines() if l.strip().startswith("{")]
