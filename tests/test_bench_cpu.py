"""bench.py's command-line contract where no GPU is needed: the reference arm (the fp64
oracle on the host cores) prints one JSON line with the keys the driver reads, ranks other
than 0 print nothing, and too few warm-up steps are refused."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def run_bench(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, BENCH, *args], capture_output=True, text=True,
                          cwd=ROOT, env=env, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    import oracle
    oracle.build()
    r = run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1", "--warmup", "3",
                   "--ref-step-budget", "0.2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny_f32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1", "--warmup", "3"],
                  env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("impl", ["ours", "reference"])
def test_too_few_warmup_steps_are_refused(impl):
    r = run_bench(["--impl", impl, "--warmup", "2"])
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr
