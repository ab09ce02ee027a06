"""bench.py's reference arm runs on the host cores alone (no GPU, no process
group) and prints one JSON line with the keys the bench contract names; under
a launcher only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    return [ln for ln in p.stdout.splitlines() if ln.strip()]


def test_reference_line_has_the_contract_keys():
    lines = run({}, "--steps", "2", "--warmup", "1", "--layers", "40")
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["unit"] == "tok/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert "2 timed layers" in d["cpu_baseline"]["sample"] and "C++ oracle" in d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]
    # a step is one layer of the stack: the per-layer time, and tok/s extrapolates it to 40 layers
    assert 0.2 * 1e3 / (40 * d["value"]) < d["ms_per_step"] < 5 * 1e3 / (40 * d["value"])


def test_other_ranks_exit_quietly():
    assert run({"RANK": "1", "WORLD_SIZE": "2"}, "--steps", "2", "--warmup", "1") == []
