"""The bench's JSON contract, checked on the reference arm (the CPU oracle),
which runs without a GPU."""

import json
import os
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]


def run_bench(*args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], capture_output=True, text=True,
                          cwd=ROOT, env=env, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = run_bench("--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", "llama3_8b_gqa",
                  "--ref-units", "4")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["value"] > 0
    assert isinstance(d["config"].get("workload"), str)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    r = run_bench("--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-units", "1",
                  env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_rejected():
    r = run_bench("--impl", "reference", "--steps", "3", "--warmup", "2")
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_default_workload_is_the_long_context_shape():
    # The headline: the largest single-GPU shape, 4 x 131,072 tokens.
    r = run_bench("--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-units", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["workload"].startswith("long_ctx_128k") and "131072" in d["config"]["workload"]
    assert d["dtype"] == "f64" and d["value"] > 0
